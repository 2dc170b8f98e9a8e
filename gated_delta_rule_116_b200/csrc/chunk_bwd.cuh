// chunk_bwd.cuh -- backward pass of the chunked KDA prefill (fp32 state and accumulation).
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
// arithmetic; 16 keeps a CTA's tiles within shared memory at d = 128). The
// dense products run on the tensor cores as warp-level tf32 tiles; the terms
// with a pairwise decay e^{g_i - g_j} (At, P and their gradients) and the 16 x 16
// triangular algebra stay on the CUDA cores, so no decay factor is ever split
// into a growing and a shrinking part. Products split over warps write their parts
// to separate buffers that are added in a fixed order (no shared-memory atomics).
// The kernels, their launch and the fp32 -> dtype casts are in chunk_bwd.cu.
#pragma once

namespace kbwd {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kC = 16;
constexpr int kNV = 64;
static_assert(kNV % 32 == 0, "whole 32-column strips");
static_assert(kC * kNV % kThreads == 0 && kC * 128 % kThreads == 0, "whole loads per thread");
constexpr float kLog2e = 1.4426950408889634f;

// Key-side rows are padded to dkp = dk rounded up to 16 (zeros past dk), so every
// product tiles into 16 x 8 blocks. Row strides are 4 floats longer than the rows
// (LD = dkp + 4, LC = C + 4, NP = NV + 4): the eight rows a warp's tensor-core
// fragment reads then start in eight different bank quads.
struct Layout {
    int dk, dkp, NV, NP, LD, LC;
    __host__ __device__ Layout(int dk_, int NV_)
        : dk(dk_), dkp((dk_ + 15) & ~15), NV(NV_), NP(NV_ + 4), LD(((dk_ + 15) & ~15) + 4), LC(kC + 4) {}
    // 12 [C][LD] tiles, 7 [C][LC], 5 [C][NP], 2 [dkp][NP], vectors, partial sums
    __host__ __device__ size_t floats() const {
        return 12ull * kC * LD + 7ull * kC * LC + 5ull * kC * NP + 2ull * dkp * NP + 3ull * dkp + 3ull * kC +
               8ull * kC * kC;
    }
};

struct Tiles {
    // Qt, Kt: q and k; Qs = q e^{g}, Ks = k e^{g}, Kh = Kb = k e^{g_C - g};
    // G: prefix sums g, in log2 units (g log2 e)
    float *Qt, *Kt, *Kh, *G, *W, *dQs, *dKb, *dW, *dKs, *dQt, *Qs, *Ks;   // [C][LD]
    float *At, *P, *X, *Tm, *dT, *dA, *dP;                      // [C][LC]
    float *V, *Up, *U, *dO, *dU;                                 // [C][NP]
    float *S, *dS;                                               // [dkp][NP]
    float *gam, *dgam, *gsum;                                    // [dkp]; gsum in log2 units
    float *bt, *dbt;                                             // [C]
    float *part;   // [8][C][C]: partial sums of At and P (three parts each) and of dT (eight)
    __device__ Tiles(float *sm, const Layout &L) {
        const int CD = kC * L.LD, CC = kC * L.LC, CN = kC * L.NP, DN = L.dkp * L.NP;
        float *p = sm;
        Qt = p; p += CD; Kt = p; p += CD; Kh = p; p += CD; G = p; p += CD; W = p; p += CD;
        dQs = p; p += CD; dKb = p; p += CD; dW = p; p += CD; dKs = p; p += CD; dQt = p; p += CD;
        Qs = p; p += CD; Ks = p; p += CD;
        At = p; p += CC; P = p; p += CC; X = p; p += CC; Tm = p; p += CC; dT = p; p += CC;
        dA = p; p += CC; dP = p; p += CC;
        V = p; p += CN; Up = p; p += CN; U = p; p += CN; dO = p; p += CN; dU = p; p += CN;
        S = p; p += DN; dS = p; p += DN;
        gam = p; p += L.dkp;
        dgam = p; p += L.dkp; gsum = p; p += L.dkp;
        bt = p; p += kC; dbt = p; p += kC; part = p;
    }
};

// ------------------------------------------------------------------ warp-level tensor-core tiles
// Products of shared-memory tiles on the tensor cores, one warp per 16 x 8 output
// block (mma.sync m16n8k8, tf32 operands, fp32 accumulation). With kSplit each
// operand x is split into tf32 parts hi(x) + lo(x) and three products are summed
// (hi hi + hi lo + lo hi), which keeps about 22 significant bits. Every product
// here takes that form, for bf16 inputs too: the gradients are differences of
// terms much larger than themselves (the gradient of k sums four such terms), and
// single tf32 products (11 bits) left errors of 6 % of a gradient element.
constexpr bool kSplitProducts = true;
// bf16 inputs (dL/dO, v) reach the products unchanged and are exact in tf32.
template <typename T> struct ExactInTf32 { static constexpr bool value = false; };
template <> struct ExactInTf32<__nv_bfloat16> { static constexpr bool value = true; };

__device__ __forceinline__ uint32_t tf32_bits(float x) { return tc::to_tf32(x) & 0xFFFFE000u; }

// d += A B for one 8-deep step; the low-part products go to e (a separate chain).
// kAExact / kBExact: that operand holds bf16 values, which tf32 represents exactly
// (its low part is zero), so its low-part product is skipped.
template <bool kSplit, bool kAExact = false, bool kBExact = false>
__device__ __forceinline__ void mma_step(float (&d)[4], float (&e)[4], const float (&a)[4],
                                         const float (&b)[2]) {
    uint32_t ah[4], bh[2];
#pragma unroll
    for (int i = 0; i < 4; ++i) ah[i] = tf32_bits(a[i]);
    bh[0] = tf32_bits(b[0]);
    bh[1] = tf32_bits(b[1]);
    if constexpr (kSplit) {
        uint32_t al[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) al[i] = tf32_bits(a[i] - __uint_as_float(ah[i]));
        const uint32_t bl0 = tf32_bits(b[0] - __uint_as_float(bh[0]));
        const uint32_t bl1 = tf32_bits(b[1] - __uint_as_float(bh[1]));
        if constexpr (!kAExact) tc::mma_16x8x8_tf32(e, al, bh[0], bh[1]);
        if constexpr (!kBExact) tc::mma_16x8x8_tf32(e, ah, bl0, bl1);
    }
    tc::mma_16x8x8_tf32(d, ah, bh[0], bh[1]);
}

// d += sum_{k0 <= k < k1} A(m, k) B(k, n) over the block at rows m0..m0+15, columns
// n0..n0+7; k1 - k0 is a multiple of 8. A and B read shared memory. Even and odd
// 8-deep steps, and the high and low parts, accumulate in separate chains.
template <bool kSplit, bool kAExact = false, bool kBExact = false, class FA, class FB>
__device__ __forceinline__ void tile_mma(float (&d)[4], const FA &A, const FB &B, int m0, int n0, int k0,
                                         int k1) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    float d1[4] = {0.f, 0.f, 0.f, 0.f}, e0[4] = {0.f, 0.f, 0.f, 0.f}, e1[4] = {0.f, 0.f, 0.f, 0.f};
    int k = k0;
    for (; k + 16 <= k1; k += 16) {
        const float a0[4] = {A(m0 + g, k + t), A(m0 + g + 8, k + t), A(m0 + g, k + t + 4),
                             A(m0 + g + 8, k + t + 4)};
        const float b0[2] = {B(k + t, n0 + g), B(k + t + 4, n0 + g)};
        const float a1[4] = {A(m0 + g, k + 8 + t), A(m0 + g + 8, k + 8 + t), A(m0 + g, k + 12 + t),
                             A(m0 + g + 8, k + 12 + t)};
        const float b1[2] = {B(k + 8 + t, n0 + g), B(k + 12 + t, n0 + g)};
        mma_step<kSplit, kAExact, kBExact>(d, e0, a0, b0);
        mma_step<kSplit, kAExact, kBExact>(d1, e1, a1, b1);
    }
    if (k < k1) {
        const float a0[4] = {A(m0 + g, k + t), A(m0 + g + 8, k + t), A(m0 + g, k + t + 4),
                             A(m0 + g + 8, k + t + 4)};
        const float b0[2] = {B(k + t, n0 + g), B(k + t + 4, n0 + g)};
        mma_step<kSplit, kAExact, kBExact>(d, e0, a0, b0);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) d[i] += d1[i] + (e0[i] + e1[i]);
}

// Visits the lane's four accumulator entries with their (row, column).
template <class F>
__device__ __forceinline__ void tile_each(float (&d)[4], int m0, int n0, const F &f) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    f(m0 + g, n0 + 2 * t, d[0]);
    f(m0 + g, n0 + 2 * t + 1, d[1]);
    f(m0 + g + 8, n0 + 2 * t, d[2]);
    f(m0 + g + 8, n0 + 2 * t + 1, d[3]);
}

// A strip of NT adjacent blocks (rows m0..m0+15, columns n0..n0+8NT-1) sharing each
// step's A fragment, whose tf32 split is then done once for the NT products:
// d[nt] += sum_{k0 <= k < k1} A(m, k) B(k, n) over block nt. Each block keeps its
// high and low products in separate chains.
template <bool kSplit, bool kAExact = false, bool kBExact = false, int NT, class FA, class FB>
__device__ __forceinline__ void strip_mma(float (&d)[NT][4], const FA &A, const FB &B, int m0, int n0,
                                          int k0, int k1) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    float e[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) e[nt][0] = e[nt][1] = e[nt][2] = e[nt][3] = 0.f;
    for (int k = k0; k < k1; k += 8) {
        const float a[4] = {A(m0 + g, k + t), A(m0 + g + 8, k + t), A(m0 + g, k + t + 4),
                            A(m0 + g + 8, k + t + 4)};
        uint32_t ah[4], al[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            ah[i] = tf32_bits(a[i]);
            al[i] = kSplit ? tf32_bits(a[i] - __uint_as_float(ah[i])) : 0u;
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const float b0 = B(k + t, n0 + 8 * nt + g), b1 = B(k + t + 4, n0 + 8 * nt + g);
            const uint32_t bh0 = tf32_bits(b0), bh1 = tf32_bits(b1);
            if constexpr (kSplit && !kAExact) tc::mma_16x8x8_tf32(e[nt], al, bh0, bh1);
            if constexpr (kSplit && !kBExact)
                tc::mma_16x8x8_tf32(e[nt], ah, tf32_bits(b0 - __uint_as_float(bh0)),
                                    tf32_bits(b1 - __uint_as_float(bh1)));
            tc::mma_16x8x8_tf32(d[nt], ah, bh0, bh1);
        }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) d[nt][i] += e[nt][i];
}

template <int NT, class F>
__device__ __forceinline__ void strip_each(float (&d)[NT][4], int m0, int n0, const F &f) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) tile_each(d[nt], m0, n0 + 8 * nt, f);
}

template <int NT>
__device__ __forceinline__ void strip_zero(float (&d)[NT][4]) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) d[nt][0] = d[nt][1] = d[nt][2] = d[nt][3] = 0.f;
}

// Strip widths: 32 value columns (kNV is a multiple of 32), 16 key channels (dkp
// is a multiple of 16).
constexpr int kVS = 4, kKS = 2;

// Brings the rows of chunk [t0, t0 + C) of q, k, log alpha, v (value slice) and, when
// given, dL/dO (value slice) and a stored state slice into L2 ahead of their loads.
template <typename Tin>
__device__ __forceinline__ void prefetch_chunk(const Tin *q, const Tin *k, const Tin *v, const float *log_alpha,
                                               const Tin *dout, const float *state, int b, int h, int T,
                                               int H, int dk, int dv, int t0, int n0) {
    const int tid = threadIdx.x;
    if (t0 < 0 || t0 >= T) return;
    const int valid = min(kC, T - t0);
    const auto pf = [](const void *p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); };
    // 128-byte lines: per token, q and k rows (dk elements), log alpha (dk floats), v and dO slices
    const int qlines = (dk * static_cast<int>(sizeof(Tin)) + 127) / 128, glines = (dk * 4 + 127) / 128;
    const int per_tok = 2 * qlines + glines + (dout ? 2 : 1);
    for (int e = tid; e < valid * per_tok; e += kThreads) {
        const int t = e / per_tok, r = e - t * per_tok;
        const long row = (static_cast<long>(b) * T + t0 + t) * H + h;
        if (r < qlines) pf(reinterpret_cast<const char *>(q + row * dk) + 128 * r);
        else if (r < 2 * qlines) pf(reinterpret_cast<const char *>(k + row * dk) + 128 * (r - qlines));
        else if (r < 2 * qlines + glines) pf(reinterpret_cast<const char *>(log_alpha + row * dk) + 128 * (r - 2 * qlines));
        else if (r == 2 * qlines + glines) pf(v + row * dv + n0);
        else pf(dout + row * dv + n0);
    }
    if (state)   // a row's slice: kNV floats from column n0, in 128-byte lines
        for (int e = tid; e < dk * (kNV / 32); e += kThreads) {
            const int c = e / (kNV / 32), l = e - c * (kNV / 32);
            if (n0 + 32 * l < dv) pf(state + static_cast<long>(c) * dv + n0 + 32 * l);
        }
}

// The state-independent terms of one chunk: g, Qs, Ks, Kb, At, P,
// X = (I + A)^{-1}, T, W = T Ks, U' = T V. Loads q, k, log alpha, v (slice), beta,
// While warp 0 solves for X, warps 1 and up run other(warp - 1): work of the
// caller's that needs none of these terms.
struct NoWork {
    __device__ void operator()(int) const {}
};
template <typename Tin, class Other = NoWork>
__device__ void chunk_terms(Tiles &s, const Layout &L, const Tin *q, const Tin *k, const Tin *v,
                            const float *log_alpha, const float *beta, int b, int h, int T, int H,
                            int dv, int t0, int valid, int n0, int nv, bool need_p,
                            const Other &other = Other()) {
    constexpr bool kSplit = kSplitProducts;
    const int tid = threadIdx.x, warp = tid >> 5, dk = L.dk, dkp = L.dkp, LD = L.LD, LC = L.LC,
              NV = L.NV, NP = L.NP;
    // every global load of the chunk is issued before the first shared-memory store
    constexpr int kPerK = kC * 128 / kThreads, kPerV = kC * kNV / kThreads;
    float qr[kPerK], kr[kPerK], gr[kPerK], vr[kPerV], br = 0.f;
#pragma unroll
    for (int u = 0; u < kPerK; ++u) {
        const int e = tid + u * kThreads, t = e / dkp, c = e - t * dkp;
        qr[u] = kr[u] = gr[u] = 0.f;
        if (e < kC * dkp && t < valid && c < dk) {
            const long o = ((static_cast<long>(b) * T + t0 + t) * H + h) * dk + c;
            qr[u] = to_f32(q[o]);
            kr[u] = to_f32(k[o]);
            gr[u] = log_alpha[o];
        }
    }
#pragma unroll
    for (int u = 0; u < kPerV; ++u) {
        const int e = tid + u * kThreads, t = e / NV, n = e - t * NV;
        vr[u] = 0.f;
        if (t < valid && n < nv) vr[u] = to_f32(v[((static_cast<long>(b) * T + t0 + t) * H + h) * dv + n0 + n]);
    }
    if (tid < valid) br = beta[(static_cast<long>(b) * T + t0 + tid) * H + h];
#pragma unroll
    for (int u = 0; u < kPerK; ++u) {
        const int e = tid + u * kThreads, t = e / dkp, c = e - t * dkp;
        if (e < kC * dkp) {
            s.Qt[t * LD + c] = qr[u];
            s.Kt[t * LD + c] = kr[u];
            s.G[t * LD + c] = gr[u];
        }
    }
#pragma unroll
    for (int u = 0; u < kPerV; ++u) {
        const int e = tid + u * kThreads, t = e / NV, n = e - t * NV;
        s.V[t * NP + n] = vr[u];
    }
    if (tid < kC) s.bt[tid] = br;
    __syncthreads();
    for (int c = tid; c < dkp; c += kThreads) {   // prefix sums (natural log), kept in log2 units
        float acc = 0.f;
        for (int t = 0; t < kC; ++t) {
            acc += s.G[t * LD + c];
            s.G[t * LD + c] = acc * kLog2e;
        }
        s.gsum[c] = acc * kLog2e;
        s.gam[c] = tc::ex2(acc * kLog2e);
    }
    __syncthreads();
    for (int e = tid; e < kC * dkp; e += kThreads) {   // Qs = q e^{g}, Ks = k e^{g}, Kb = k e^{g_C - g}
        const int t = e / dkp, c = e - t * dkp;
        const float gv = s.G[t * LD + c];
        const float up = tc::ex2(gv), down = tc::ex2(s.gsum[c] - gv);
        const float kv = s.Kt[t * LD + c];
        s.Qs[t * LD + c] = s.Qt[t * LD + c] * up;
        s.Ks[t * LD + c] = kv * up;
        s.Kh[t * LD + c] = kv * down;
    }
    // At (strict lower) and P (lower): one thread per (pair i >= j, third of the
    // channels), partial sums written apart and added in a fixed order below; both use
    // the same pairwise decays e^{g_i - g_j} <= 1
    {
        constexpr int kPairs = kC * (kC + 1) / 2;
        static_assert(3 * kPairs <= kThreads, "one pass over the items");
        const int n4 = dkp / 4;
        if (tid < 3 * kPairs) {
            const int part = tid / kPairs, p = tid - part * kPairs;
            int i = static_cast<int>((sqrtf(8.f * p + 1.f) - 1.f) * 0.5f);   // p = i (i + 1) / 2 + j
            if ((i + 1) * (i + 2) / 2 <= p) ++i;
            if (i * (i + 1) / 2 > p) --i;
            const int j = p - i * (i + 1) / 2;
            const float4 *ki = reinterpret_cast<const float4 *>(s.Kt + i * LD);
            const float4 *kj = reinterpret_cast<const float4 *>(s.Kt + j * LD);
            const float4 *qi = reinterpret_cast<const float4 *>(s.Qt + i * LD);
            const float4 *gi = reinterpret_cast<const float4 *>(s.G + i * LD);
            const float4 *gj = reinterpret_cast<const float4 *>(s.G + j * LD);
            float at[4] = {0.f, 0.f, 0.f, 0.f}, pp[4] = {0.f, 0.f, 0.f, 0.f};
            const int c4a = part * n4 / 3, c4b = (part + 1) * n4 / 3;
            if (need_p) {
                for (int c4 = c4a; c4 < c4b; ++c4) {
                    const float4 a = ki[c4], bj = kj[c4], q4 = qi[c4], x = gi[c4], y = gj[c4];
                    const float w0 = bj.x * tc::ex2(x.x - y.x), w1 = bj.y * tc::ex2(x.y - y.y);
                    const float w2 = bj.z * tc::ex2(x.z - y.z), w3 = bj.w * tc::ex2(x.w - y.w);
                    at[0] = fmaf(a.x, w0, at[0]); at[1] = fmaf(a.y, w1, at[1]);
                    at[2] = fmaf(a.z, w2, at[2]); at[3] = fmaf(a.w, w3, at[3]);
                    pp[0] = fmaf(q4.x, w0, pp[0]); pp[1] = fmaf(q4.y, w1, pp[1]);
                    pp[2] = fmaf(q4.z, w2, pp[2]); pp[3] = fmaf(q4.w, w3, pp[3]);
                }
            } else {
                for (int c4 = c4a; c4 < c4b; ++c4) {
                    const float4 a = ki[c4], bj = kj[c4], x = gi[c4], y = gj[c4];
                    at[0] = fmaf(a.x, bj.x * tc::ex2(x.x - y.x), at[0]);
                    at[1] = fmaf(a.y, bj.y * tc::ex2(x.y - y.y), at[1]);
                    at[2] = fmaf(a.z, bj.z * tc::ex2(x.z - y.z), at[2]);
                    at[3] = fmaf(a.w, bj.w * tc::ex2(x.w - y.w), at[3]);
                }
            }
            float *part_out = s.part + part * 2 * kC * kC + i * kC + j;   // [part][At|P][i][j]
            part_out[0] = (at[0] + at[1]) + (at[2] + at[3]);
            part_out[kC * kC] = (pp[0] + pp[1]) + (pp[2] + pp[3]);
        }
    }
    __syncthreads();
    static_assert(kThreads - 32 >= kC * kC, "P in one pass of warps 1 and up");
    const auto third = [&](int which, int e) {   // the three partial sums of At or P, in order
        const float *x = s.part + which * kC * kC + e;
        return (x[0] + x[2 * kC * kC]) + x[4 * kC * kC];
    };
    if (warp > 0) {
        if (tid - 32 < kC * kC) {
            const int e = tid - 32, i = e / kC, j = e - i * kC;
            s.P[i * LC + j] = (need_p && j <= i) ? third(1, e) : 0.f;
        }
        other(warp - 1);
    } else {
        for (int e = tid; e < kC * kC; e += 32) {
            const int i = e / kC, j = e - i * kC;
            s.At[i * LC + j] = j < i ? third(0, e) : 0.f;
        }
        __syncwarp();
    }
    if (warp == 0) {
        // X = (I + A)^{-1}, A = Diag(beta) At, in 8 x 8 blocks: the two diagonal blocks
        // X00 = (I + A00)^{-1} and X11 = (I + A11)^{-1} by forward substitution (lane l < 16
        // takes column l % 8 of block l / 8), then X10 = -X11 (A10 X00) through dA, which
        // is free until the gradient terms; X01 = 0. T = X Diag(beta).
        static_assert(kC == 16, "two 8 x 8 diagonal blocks");
        const int lane = tid & 31;
        if (lane < kC) {
            const int o = (lane >> 3) * 8, jj = lane & 7;
            float xc[8];   // column jj of the diagonal block, in registers
#pragma unroll
            for (int ii = 0; ii < 8; ++ii) {
                float acc = 0.f;
#pragma unroll
                for (int mm = 0; mm < ii; ++mm) acc = fmaf(s.At[(o + ii) * LC + o + mm], xc[mm], acc);
                xc[ii] = ii == jj ? 1.f : (ii > jj ? -s.bt[o + ii] * acc : 0.f);   // xc[mm] = 0 for mm < jj
                s.X[(o + ii) * LC + o + jj] = xc[ii];
                if (o == 8) s.X[ii * LC + 8 + jj] = 0.f;   // X01 = 0
            }
        }
        __syncwarp();
#pragma unroll
        for (int r = 0; r < 2; ++r) {   // Y = A10 X00 = Diag(beta_8..15) At[8..15][0..7] X00
            const int e = lane + 32 * r, m = e >> 3, j = e & 7;
            float acc = 0.f;
            for (int n = j; n < 8; ++n) acc = fmaf(s.At[(8 + m) * LC + n], s.X[n * LC + j], acc);
            s.dA[m * LC + j] = s.bt[8 + m] * acc;
        }
        __syncwarp();
#pragma unroll
        for (int r = 0; r < 2; ++r) {   // X10 = -X11 Y
            const int e = lane + 32 * r, i = e >> 3, j = e & 7;
            float acc = 0.f;
            for (int m = 0; m <= i; ++m) acc = fmaf(s.X[(8 + i) * LC + 8 + m], s.dA[m * LC + j], acc);
            s.X[(8 + i) * LC + j] = -acc;
        }
        __syncwarp();
        for (int e = lane; e < kC * kC; e += 32) {
            const int i = e / kC, j = e - i * kC;
            s.Tm[i * LC + j] = s.X[i * LC + j] * s.bt[j];
        }
    }
    __syncthreads();
    {   // W = T Ks (16-channel strips), U' = T V (32-column strips); T is lower triangular
        const int nW = dkp / 16, nU = NV / 32;
        const auto A = [&](int m, int kk) { return s.Tm[m * LC + kk]; };
        for (int tl = warp; tl < nW + nU; tl += kWarps) {
            if (tl < nW) {
                float d[kKS][4];
                strip_zero(d);
                strip_mma<kSplit>(d, A, [&](int kk, int n) { return s.Ks[kk * LD + n]; }, 0, tl * 16, 0, kC);
                strip_each(d, 0, tl * 16, [&](int r, int c, float &x) { s.W[r * LD + c] = x; });
            } else {
                float d[kVS][4];
                strip_zero(d);
                const int j0 = (tl - nW) * 32;
                strip_mma<kSplit, false, ExactInTf32<Tin>::value>(
                    d, A, [&](int kk, int n) { return s.V[kk * NP + n]; }, 0, j0, 0, kC);
                strip_each(d, 0, j0, [&](int r, int c, float &x) { s.Up[r * NP + c] = x; });
            }
        }
    }
    __syncthreads();
}

// Bounds of part p of `parts` of a depth of k8 8-deep steps (parts may be empty).
__device__ __forceinline__ int depth_lo(int p, int k8, int parts) { return (p * k8) / parts * 8; }

// U = U' - W S, full depth, one warp per 8 value columns.
template <bool kSplit>
__device__ __forceinline__ void u_block(Tiles &s, const Layout &L, int j0) {
    const int LD = L.LD, NP = L.NP;
    float d[4];
    tile_each(d, 0, j0, [&](int r, int c, float &x) { x = s.Up[r * NP + c]; });
    tile_mma<kSplit>(d, [&](int m, int kk) { return -s.W[m * LD + kk]; },
                     [&](int kk, int n) { return s.S[kk * NP + n]; }, 0, j0, 0, L.dkp);
    tile_each(d, 0, j0, [&](int r, int c, float &x) { s.U[r * NP + c] = x; });
}

// S <- Diag(gamma) S + Kb^T U over 16-row x 32-column strips.
template <bool kSplit>
__device__ __forceinline__ void state_update(Tiles &s, const Layout &L) {
    const int warp = threadIdx.x >> 5, LD = L.LD, NP = L.NP, nN = L.NV / 32;
    for (int tl = warp; tl < (L.dkp / 16) * nN; tl += kWarps) {
        const int m0 = (tl / nN) * 16, j0 = (tl - (tl / nN) * nN) * 32;
        float d[kVS][4];
        strip_each(d, m0, j0, [&](int r, int c, float &x) { x = s.gam[r] * s.S[r * NP + c]; });
        strip_mma<kSplit>(d, [&](int m, int kk) { return s.Kh[kk * LD + m]; },
                          [&](int kk, int n) { return s.U[kk * NP + n]; }, m0, j0, 0, kC);
        strip_each(d, m0, j0, [&](int r, int c, float &x) { s.S[r * NP + c] = x; });
    }
}

// Forward chain storing the entry state of every chunk: states[bh][chunk][dk][dv].
template <typename Tin>
__device__ void states_body(float *sm, const Tin *q, const Tin *k, const Tin *v, const float *log_alpha,
                            const float *beta, const float *S0, float *states, int T, int H, int dk,
                            int dv) {
    constexpr bool kSplit = kSplitProducts;
    const Layout L(dk, kNV);
    Tiles s(sm, L);
    const int tid = threadIdx.x, warp = tid >> 5, dkp = L.dkp, NV = L.NV, NP = L.NP;
    const int bh = blockIdx.x, b = bh / H, h = bh - b * H;
    const int n0 = blockIdx.y * NV, nv = min(NV, dv - n0);
    const int nchunks = (T + kC - 1) / kC;
    for (int e = tid; e < dkp * NV; e += kThreads) {
        const int c = e / NV, n = e - c * NV;
        s.S[c * NP + n] = (S0 && c < dk && n < nv) ? S0[(static_cast<long>(bh) * dk + c) * dv + n0 + n] : 0.f;
    }
    for (int ch = 0; ch < nchunks; ++ch) {
        const int t0 = ch * kC, valid = min(kC, T - t0);
        __syncthreads();
        float *dst = states + (static_cast<long>(bh) * nchunks + ch) * dk * dv;
        prefetch_chunk<Tin>(q, k, v, log_alpha, nullptr, nullptr, b, h, T, H, dk, dv, t0 + kC, n0);
        // the chunk's entry state goes out while warp 0 solves for X
        chunk_terms(s, L, q, k, v, log_alpha, beta, b, h, T, H, dv, t0, valid, n0, nv, false, [&](int w) {
            for (int e = w * 32 + (tid & 31); e < dk * NV; e += kThreads - 32) {
                const int c = e / NV, n = e - c * NV;
                if (n < nv) dst[static_cast<long>(c) * dv + n0 + n] = s.S[c * NP + n];
            }
        });
        for (int tl = warp; tl < NV / 8; tl += kWarps) u_block<kSplit>(s, L, tl * 8);   // U = U' - W S
        __syncthreads();
        state_update<kSplit>(s, L);   // S <- Diag(gamma) S + Kb^T U
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
    constexpr bool kSplit = kSplitProducts;
    const Layout L(dk, kNV);
    Tiles s(sm, L);
    const int tid = threadIdx.x, warp = tid >> 5, dkp = L.dkp, LD = L.LD, LC = L.LC, NV = L.NV,
              NP = L.NP;
    const int bh = blockIdx.x, b = bh / H, h = bh - b * H;
    const int n0 = blockIdx.y * NV, nv = min(NV, dv - n0);
    const int nchunks = (T + kC - 1) / kC;
    const int nU = NV / 32, nQ = dkp / 16, nS = (dkp / 16) * nU;   // strip counts
    for (int e = tid; e < dkp * NV; e += kThreads) {
        const int c = e / NV, n = e - c * NV;
        s.dS[c * NP + n] =
            (dS_T && c < dk && n < nv) ? dS_T[(static_cast<long>(bh) * dk + c) * dv + n0 + n] : 0.f;
    }
    for (int ch = nchunks - 1; ch >= 0; --ch) {
        const int t0 = ch * kC, valid = min(kC, T - t0);
        __syncthreads();
        if (ch > 0)
            prefetch_chunk<Tin>(q, k, v, log_alpha, dout,
                                states + (static_cast<long>(bh) * nchunks + ch - 1) * dk * dv, b, h, T, H,
                                dk, dv, t0 - kC, n0);
        {   // the chunk's entry state and dL/dO, all loads issued before the stores
            const float *src = states + (static_cast<long>(bh) * nchunks + ch) * dk * dv;
            constexpr int kPerS = 128 * kNV / kThreads, kPerO = kC * kNV / kThreads;
            float sr[kPerS], orr[kPerO];
#pragma unroll
            for (int u = 0; u < kPerS; ++u) {
                const int e = tid + u * kThreads, c = e / NV, n = e - c * NV;
                sr[u] = (c < dk && n < nv) ? src[static_cast<long>(c) * dv + n0 + n] : 0.f;
            }
#pragma unroll
            for (int u = 0; u < kPerO; ++u) {
                const int e = tid + u * kThreads, t = e / NV, n = e - t * NV;
                orr[u] = (t < valid && n < nv)
                             ? to_f32(dout[((static_cast<long>(b) * T + t0 + t) * H + h) * dv + n0 + n])
                             : 0.f;
            }
#pragma unroll
            for (int u = 0; u < kPerS; ++u) {
                const int e = tid + u * kThreads, c = e / NV, n = e - c * NV;
                if (c < dkp) s.S[c * NP + n] = sr[u];
            }
#pragma unroll
            for (int u = 0; u < kPerO; ++u) {
                const int e = tid + u * kThreads, t = e / NV, n = e - t * NV;
                s.dO[t * NP + n] = orr[u];
            }
        }
        // While warp 0 solves for X: gamma's gradient (through the state decay, warps 1-4,
        // one state row per thread) and dQs = dO S^T (warps 5 and up)
        chunk_terms(s, L, q, k, v, log_alpha, beta, b, h, T, H, dv, t0, valid, n0, nv, true, [&](int w) {
            if (w < 4) {
                const int c = w * 32 + (tid & 31);
                if (c < dkp) {
                    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
                    for (int n = 0; n < NV; n += 4) {
                        a0 = fmaf(s.dS[c * NP + n], s.S[c * NP + n], a0);
                        a1 = fmaf(s.dS[c * NP + n + 1], s.S[c * NP + n + 1], a1);
                        a2 = fmaf(s.dS[c * NP + n + 2], s.S[c * NP + n + 2], a2);
                        a3 = fmaf(s.dS[c * NP + n + 3], s.S[c * NP + n + 3], a3);
                    }
                    s.dgam[c] = ((a0 + a1) + (a2 + a3)) * s.gam[c];
                }
            } else {
                for (int tl = w - 4; tl < nQ; tl += kWarps - 5) {
                    const int c0 = tl * 16;
                    float d[kKS][4];
                    strip_zero(d);
                    strip_mma<kSplit, ExactInTf32<Tin>::value>(d, [&](int m, int kk) { return s.dO[m * NP + kk]; },
                                      [&](int kk, int c) { return s.S[c * NP + kk]; }, 0, c0, 0, NV);
                    strip_each(d, 0, c0, [&](int r, int c, float &x) { s.dQs[r * LD + c] = x; });
                }
            }
        });
        for (int tl = warp; tl < NV / 8; tl += kWarps) u_block<kSplit>(s, L, tl * 8);   // U = U' - W S
        __syncthreads();
        // dU = P^T dO + Kb dS (full depth, 8-column blocks); dKb = U dS^T
        for (int tl = warp; tl < NV / 8 + nQ; tl += kWarps) {
            if (tl < NV / 8) {
                const int j0 = tl * 8;
                float d[4] = {0.f, 0.f, 0.f, 0.f};
                tile_mma<kSplit, false, ExactInTf32<Tin>::value>(d, [&](int m, int kk) { return s.P[kk * LC + m]; },
                                 [&](int kk, int n) { return s.dO[kk * NP + n]; }, 0, j0, 0, kC);
                tile_mma<kSplit>(d, [&](int m, int kk) { return s.Kh[m * LD + kk]; },
                                 [&](int kk, int n) { return s.dS[kk * NP + n]; }, 0, j0, 0, dkp);
                tile_each(d, 0, j0, [&](int r, int c, float &x) { s.dU[r * NP + c] = x; });
            } else {
                const int c0 = (tl - NV / 8) * 16;
                float d[kKS][4];
                strip_zero(d);
                strip_mma<kSplit>(d, [&](int m, int kk) { return s.U[m * NP + kk]; },
                                  [&](int kk, int c) { return s.dS[c * NP + kk]; }, 0, c0, 0, NV);
                strip_each(d, 0, c0, [&](int r, int c, float &x) { s.dKb[r * LD + c] = x; });
            }
        }
        __syncthreads();
        // dS <- Diag(gamma) dS + Qs^T dO - W^T dU (in place: each strip reads only its own
        // dS entries); dW = -dU S^T; dV = T^T dU
        for (int tl = warp; tl < nS + nQ + nU; tl += kWarps) {
            if (tl < nS) {
                const int m0 = (tl / nU) * 16, j0 = (tl - (tl / nU) * nU) * 32;
                float d[kVS][4];
                strip_each(d, m0, j0, [&](int r, int c, float &x) { x = s.gam[r] * s.dS[r * NP + c]; });
                strip_mma<kSplit, false, ExactInTf32<Tin>::value>(d, [&](int m, int kk) { return s.Qs[kk * LD + m]; },
                                  [&](int kk, int n) { return s.dO[kk * NP + n]; }, m0, j0, 0, kC);
                strip_mma<kSplit>(d, [&](int m, int kk) { return -s.W[kk * LD + m]; },
                                  [&](int kk, int n) { return s.dU[kk * NP + n]; }, m0, j0, 0, kC);
                strip_each(d, m0, j0, [&](int r, int c, float &x) { s.dS[r * NP + c] = x; });
            } else if (tl < nS + nQ) {
                const int c0 = (tl - nS) * 16;
                float d[kKS][4];
                strip_zero(d);
                strip_mma<kSplit>(d, [&](int m, int kk) { return -s.dU[m * NP + kk]; },
                                  [&](int kk, int c) { return s.S[c * NP + kk]; }, 0, c0, 0, NV);
                strip_each(d, 0, c0, [&](int r, int c, float &x) { s.dW[r * LD + c] = x; });
            } else {
                const int j0 = (tl - nS - nQ) * 32;
                float d[kVS][4];
                strip_zero(d);
                strip_mma<kSplit>(d, [&](int m, int kk) { return s.Tm[kk * LC + m]; },
                                  [&](int kk, int n) { return s.dU[kk * NP + n]; }, 0, j0, 0, kC);
                strip_each(d, 0, j0, [&](int r, int c, float &x) {
                    if (r < valid && c < nv)
                        dv_out[((static_cast<long>(b) * T + t0 + r) * H + h) * dv + n0 + c] = from_f32<Tin>(x);
                });
            }
        }
        __syncthreads();
        // dT = dW Ks^T + dU V^T, both depths split in eight parts written apart and summed
        // in order below; its upper triangle is masked where it is read.
        // dP = lower(dO U^T); dKs = T^T dW.
        for (int tl = warp; tl < 9 + nQ; tl += kWarps) {
            float d[kKS][4];
            strip_zero(d);
            if (tl < 8) {
                strip_mma<kSplit>(d, [&](int m, int kk) { return s.dW[m * LD + kk]; },
                                  [&](int kk, int j) { return s.Ks[j * LD + kk]; }, 0, 0,
                                  depth_lo(tl, dkp / 8, 8), depth_lo(tl + 1, dkp / 8, 8));
                strip_mma<kSplit, false, ExactInTf32<Tin>::value>(d, [&](int m, int kk) { return s.dU[m * NP + kk]; },
                                  [&](int kk, int j) { return s.V[j * NP + kk]; }, 0, 0,
                                  depth_lo(tl, NV / 8, 8), depth_lo(tl + 1, NV / 8, 8));
                strip_each(d, 0, 0, [&](int r, int c, float &x) { s.part[tl * kC * kC + r * kC + c] = x; });
            } else if (tl == 8) {
                strip_mma<kSplit, ExactInTf32<Tin>::value>(d, [&](int m, int kk) { return s.dO[m * NP + kk]; },
                                  [&](int kk, int j) { return s.U[j * NP + kk]; }, 0, 0, 0, NV);
                strip_each(d, 0, 0, [&](int r, int c, float &x) { s.dP[r * LC + c] = c <= r ? x : 0.f; });
            } else {
                const int c0 = (tl - 9) * 16;
                strip_mma<kSplit>(d, [&](int m, int kk) { return s.Tm[kk * LC + m]; },
                                  [&](int kk, int c) { return s.dW[kk * LD + c]; }, 0, c0, 0, kC);
                strip_each(d, 0, c0, [&](int r, int c, float &x) { s.dKs[r * LD + c] = x; });
            }
        }
        __syncthreads();
        for (int e = tid; e < kC * kC; e += kThreads) {
            const float *x = s.part + e;
            float a = 0.f;
#pragma unroll
            for (int part = 0; part < 8; ++part) a += x[part * kC * kC];
            s.dT[(e / kC) * LC + e % kC] = a;
        }
        __syncthreads();
        // Z = X^T dX with dX = lower(dT) Diag(beta) (kept in dA), and dbeta's T part
        for (int e = tid; e < kC * kC + kC; e += kThreads) {
            if (e < kC * kC) {
                const int i = e / kC, bcol = e - i * kC;
                float acc = 0.f;
                for (int a = max(i, bcol); a < kC; ++a) acc = fmaf(s.X[a * LC + i], s.dT[a * LC + bcol], acc);
                s.dA[i * LC + bcol] = acc * s.bt[bcol];
            } else {
                const int j = e - kC * kC;
                float acc = 0.f;
                for (int i = j; i < kC; ++i) acc = fmaf(s.dT[i * LC + j], s.X[i * LC + j], acc);
                s.dbt[j] = acc;
            }
        }
        __syncthreads();
        // dA = -strict_lower(Z X^T); dbeta's A part (row sums of dA o At, over the 16
        // lanes that hold a row); dAt = Diag(beta) dA, into dT
        static_assert(kC == 16 && kThreads >= kC * kC, "a row of dA per half warp");
        if (tid < kC * kC) {
            const int i = tid / kC, j = tid - i * kC;
            float acc = 0.f;
            if (j < i)
                for (int bcol = 0; bcol <= j; ++bcol) acc = fmaf(s.dA[i * LC + bcol], s.X[j * LC + bcol], acc);
            float r = -acc * s.At[i * LC + j];
            r += __shfl_xor_sync(0xffffffffu, r, 8);
            r += __shfl_xor_sync(0xffffffffu, r, 4);
            r += __shfl_xor_sync(0xffffffffu, r, 2);
            r += __shfl_xor_sync(0xffffffffu, r, 1);
            if (j == 0) s.dbt[i] += r;
            s.dT[i * LC + j] = -acc * s.bt[i];
        }
        __syncthreads();
        // The intra-chunk products, term by term (E_ij = e^{g_i - g_j} per channel):
        //   R_i  = sum_{j<i}  dAt_ij k_j E_ij             (row side of A,   into dW)
        //   Cc_j = sum_{i>j}  dAt_ij k_i E_ij
        //        + sum_{i>=j} dP_ij  q_i E_ij             (column side)
        //   Rq_i = sum_{j<=i} dP_ij  k_j E_ij             (row side of P,   into dQt)
        // Each decay is computed once for the three sums: a warp takes the rows i of one
        // residue mod 4 and 32 channels (a lane per channel), walks the pairs j < i of its
        // rows, writes R and Rq of those rows and writes its part of every Cc into the
        // S tile (S is not read again in this chunk); the four parts are added in order
        // where Cc is used. The diagonal (E = 1) starts Rq and Cc.
        {
            const int part = warp & 3, c = (warp >> 2) * 32 + (tid & 31);
            static_assert(kWarps == 16, "four residues x four groups of 32 channels");
            if (c < dkp) {
                float g[kC], kk[kC], qq[kC], Cc[kC];
#pragma unroll
                for (int i = 0; i < kC; ++i) {
                    g[i] = s.G[i * LD + c];
                    kk[i] = s.Kt[i * LD + c];
                    qq[i] = s.Qt[i * LD + c];
                    Cc[i] = (i & 3) == part ? s.dP[i * LC + i] * qq[i] : 0.f;
                }
#pragma unroll
                for (int i = 0; i < kC; ++i) {
                    if ((i & 3) != part) continue;
                    float R = 0.f, Rq = s.dP[i * LC + i] * kk[i];
#pragma unroll
                    for (int j = 0; j < i; ++j) {
                        const float E = tc::ex2(g[i] - g[j]);
                        const float a = s.dT[i * LC + j], p = s.dP[i * LC + j];
                        R = fmaf(a * kk[j], E, R);
                        Rq = fmaf(p * kk[j], E, Rq);
                        Cc[j] = fmaf(fmaf(a, kk[i], p * qq[i]), E, Cc[j]);
                    }
                    s.dW[i * LD + c] = R;
                    s.dQt[i * LD + c] = Rq;
                }
#pragma unroll
                for (int j = 0; j < kC; ++j) s.S[(part * kC + j) * dkp + c] = Cc[j];
            }
        }
        __syncthreads();
        // dk, dq; dg per token and channel (into dKs, after its use)
        for (int e = tid; e < kC * dkp; e += kThreads) {
            const int t = e / dkp, c = e - t * dkp;
            const float gv = s.G[t * LD + c];
            const float up = tc::ex2(gv), down = tc::ex2(s.gsum[c] - gv);
            const float kv = s.Kt[t * LD + c], qv = s.Qt[t * LD + c];
            const float *ccp = s.S + t * dkp + c;   // the four parts of Cc, in order
            const float cc = ((ccp[0] + ccp[kC * dkp]) + ccp[2 * kC * dkp]) + ccp[3 * kC * dkp];
            const float rk = s.dW[t * LD + c], rq = s.dQt[t * LD + c];
            const float dks = s.dKs[t * LD + c], dkb = s.dKb[t * LD + c], dqs = s.dQs[t * LD + c];
            const float dk_v = rk + cc + dks * up + dkb * down;
            const float dq_v = rq + dqs * up;
            const float dg = kv * (rk - cc) + qv * rq + dks * s.Ks[t * LD + c] + dqs * s.Qs[t * LD + c] -
                             dkb * s.Kh[t * LD + c];
            s.dKs[t * LD + c] = dg;
            if (t < valid && c < dk) {
                const long o = ((static_cast<long>(b) * T + t0 + t) * H + h) * dk + c;
                atomicAdd(dk_acc + o, dk_v);
                atomicAdd(dq_acc + o, dq_v);
            }
        }
        __syncthreads();
        static_assert(kThreads >= 4 * 128, "four threads per channel");
        {   // g_C's own terms, then the in-chunk suffix sums: four threads per channel, four
            // tokens each, the parts' totals combined across the four lanes
            const int c = tid >> 2, part = tid & 3;
            float gc = 0.f, loc = 0.f, sfx[4];
            if (c < dkp) {
#pragma unroll
                for (int u = 3; u >= 0; --u) {
                    const int t = 4 * part + u;
                    gc = fmaf(s.dKb[t * LD + c], s.Kh[t * LD + c], gc);
                    loc += s.dKs[t * LD + c];
                    sfx[u] = loc;
                }
            }
            gc += __shfl_xor_sync(0xffffffffu, gc, 1);
            gc += __shfl_xor_sync(0xffffffffu, gc, 2);
            // tokens after this part's: the totals of the higher parts
            const float t1 = __shfl_down_sync(0xffffffffu, loc, 1), t2 = __shfl_down_sync(0xffffffffu, loc, 2),
                        t3 = __shfl_down_sync(0xffffffffu, loc, 3);
            const float after = (part < 3 ? t1 : 0.f) + (part < 2 ? t2 : 0.f) + (part < 1 ? t3 : 0.f);
            if (c < dk) {
                const float base = (c < dkp ? s.dgam[c] : 0.f) + gc + after;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int t = 4 * part + u;
                    if (t < valid)
                        atomicAdd(dlog_alpha + ((static_cast<long>(b) * T + t0 + t) * H + h) * dk + c, base + sfx[u]);
                }
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
