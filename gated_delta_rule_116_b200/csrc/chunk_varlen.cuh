// chunk_varlen.cuh -- chunked KDA prefill over a packed batch of variable-length
// sequences, fp32 on CUDA cores (bodies; kernels and launch in chunk_varlen.cu).
//
// Sequence n occupies tokens cu_seqlens[n] .. cu_seqlens[n+1]-1 of packed
// [total_T, H, d] tensors and starts from its own state (or zeros); the
// recurrence never crosses a sequence boundary. With a slot map, sequence n's
// initial and final states are row slot[n] of state caches [slots, H, dk, dv]
// (the layout of the decode step's cache, so a prefill can fill the rows that
// decode steps then continue, in place); without one, row n. Per sequence this is the
// chunked form of the prefill (Kimi Linear summary, es.news.hada.io/topic?id=31936,
// section "Algoritmo paralelo por chunks"): fixed-length chunks starting from
// the previous chunk's last state, the WY/UT form, and outputs that add the
// inter-chunk recurrent part to the intra-chunk parallel part. The chunk terms
// are those of the backward pass (chunk_bwd.cuh: chunk_terms), 16 tokens long;
// a CTA owns (sequence, head, 32 value columns).
#pragma once

namespace kvar {

using kbwd::kC;
using kbwd::kNV;
using kbwd::kThreads;

template <typename Tin>
__device__ void varlen_body(float *sm, const Tin *q, const Tin *k, const Tin *v, const float *log_alpha,
                            const float *beta, const int32_t *cu_seqlens, const int32_t *slot,
                            const float *S0, Tin *out, float *S_T, int total_T, int H, int dk,
                            int dv) {
    const kbwd::Layout L(dk, kNV);
    kbwd::Tiles s(sm, L);
    const int tid = threadIdx.x, LD = L.LD, LC = L.LC, NV = L.NV, NP = L.NP;
    const int nh = blockIdx.x, n = nh / H, h = nh - n * H;
    const int n0 = blockIdx.y * NV, nv = min(NV, dv - n0);
    // the offsets are device data: clamp them so that every access stays in [0, total_T)
    const int start = min(max(cu_seqlens[n], 0), total_T);
    const int end = min(max(cu_seqlens[n + 1], start), total_T);
    const int len = end - start;
    const long row = (slot ? static_cast<long>(slot[n]) : static_cast<long>(n)) * H + h;   // state row
    for (int e = tid; e < dk * NV; e += kThreads) {
        const int c = e / NV, j = e - c * NV;
        s.S[c * NP + j] = (S0 && j < nv) ? S0[(row * dk + c) * dv + n0 + j] : 0.f;
    }
    const int nchunks = (len + kC - 1) / kC;
    for (int ch = 0; ch < nchunks; ++ch) {
        const int t0 = start + ch * kC, valid = min(kC, end - t0);
        __syncthreads();
        kbwd::chunk_terms(s, L, q, k, v, log_alpha, beta, 0, h, total_T, H, dv, t0, valid, n0, nv, true);
        for (int e = tid; e < kC * NV; e += kThreads) {   // U = U' - W S
            const int i = e / NV, j = e - i * NV;
            float acc = s.Up[i * NP + j];
            for (int c = 0; c < dk; ++c) acc = fmaf(-s.W[i * LD + c], s.S[c * NP + j], acc);
            s.U[i * NP + j] = acc;
        }
        __syncthreads();
        for (int e = tid; e < kC * NV; e += kThreads) {   // O = Qs S + P U
            const int i = e / NV, j = e - i * NV;
            if (i >= valid || j >= nv) continue;
            float acc = 0.f;
            for (int c = 0; c < dk; ++c) acc = fmaf(s.Qs[i * LD + c], s.S[c * NP + j], acc);
            for (int m = 0; m <= i; ++m) acc = fmaf(s.P[i * LC + m], s.U[m * NP + j], acc);
            out[(static_cast<long>(t0 + i) * H + h) * dv + n0 + j] = from_f32<Tin>(acc);
        }
        __syncthreads();
        for (int e = tid; e < dk * NV; e += kThreads) {   // S <- Diag(gamma) S + Kb^T U
            const int c = e / NV, j = e - c * NV;
            float acc = s.gam[c] * s.S[c * NP + j];
            for (int t = 0; t < kC; ++t) acc = fmaf(s.Kh[t * LD + c], s.U[t * NP + j], acc);
            s.S[c * NP + j] = acc;
        }
    }
    __syncthreads();
    if (S_T)
        for (int e = tid; e < dk * NV; e += kThreads) {
            const int c = e / NV, j = e - c * NV;
            if (j < nv) S_T[(row * dk + c) * dv + n0 + j] = s.S[c * NP + j];
        }
}

}  // namespace kvar
