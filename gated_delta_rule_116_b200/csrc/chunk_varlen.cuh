// chunk_varlen.cuh -- chunked KDA prefill over a packed batch of variable-length
// sequences, fp32 state, products on the tensor cores through warp-level tf32 tiles (bodies;
// kernels and launch in chunk_varlen.cu).
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
// a CTA owns (sequence, head, 64 value columns).
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
    constexpr bool kSplit = kbwd::kSplitProducts;
    const kbwd::Layout L(dk, kNV);
    kbwd::Tiles s(sm, L);
    const int tid = threadIdx.x, warp = tid >> 5, dkp = L.dkp, LD = L.LD, LC = L.LC, NV = L.NV,
              NP = L.NP;
    const int nh = blockIdx.x, n = nh / H, h = nh - n * H;
    const int n0 = blockIdx.y * NV, nv = min(NV, dv - n0);
    // the offsets are device data: clamp them so that every access stays in [0, total_T)
    const int start = min(max(cu_seqlens[n], 0), total_T);
    const int end = min(max(cu_seqlens[n + 1], start), total_T);
    const int len = end - start;
    const long row = (slot ? static_cast<long>(slot[n]) : static_cast<long>(n)) * H + h;   // state row
    const int nU = NV / 8;
    static_assert(2 * (kNV / 8) <= kbwd::kWarps, "one output block per warp");
    for (int e = tid; e < dkp * NV; e += kThreads) {
        const int c = e / NV, j = e - c * NV;
        s.S[c * NP + j] = (S0 && c < dk && j < nv) ? S0[(row * dk + c) * dv + n0 + j] : 0.f;
    }
    const int nchunks = (len + kC - 1) / kC;
    for (int ch = 0; ch < nchunks; ++ch) {
        const int t0 = start + ch * kC, valid = min(kC, end - t0);
        __syncthreads();
        kbwd::chunk_terms(s, L, q, k, v, log_alpha, beta, 0, h, total_T, H, dv, t0, valid, n0, nv, true);
        // U = U' - W S (warps 0 .. nU-1); the inter-chunk part of O, Qs S (warps nU .. 2nU-1)
        float od[4] = {0.f, 0.f, 0.f, 0.f};
        const int oj0 = (warp - nU) * 8;
        if (warp < nU) {
            kbwd::u_block<kSplit>(s, L, warp * 8);
        } else if (warp < 2 * nU) {
            kbwd::tile_mma<kSplit>(od, [&](int m, int kk) { return s.Qs[m * LD + kk]; },
                                   [&](int kk, int j) { return s.S[kk * NP + j]; }, 0, oj0, 0, dkp);
        }
        __syncthreads();
        if (warp >= nU && warp < 2 * nU) {   // O += P U, written out
            kbwd::tile_mma<kSplit>(od, [&](int m, int kk) { return s.P[m * LC + kk]; },
                                   [&](int kk, int j) { return s.U[kk * NP + j]; }, 0, oj0, 0, kC);
            kbwd::tile_each(od, 0, oj0, [&](int i, int j, float &x) {
                if (i < valid && j < nv) out[(static_cast<long>(t0 + i) * H + h) * dv + n0 + j] = from_f32<Tin>(x);
            });
        }
        kbwd::state_update<kSplit>(s, L);   // S <- Diag(gamma) S + Kb^T U
    }
    __syncthreads();
    if (S_T)
        for (int e = tid; e < dk * NV; e += kThreads) {
            const int c = e / NV, j = e - c * NV;
            if (j < nv) S_T[(row * dk + c) * dv + n0 + j] = s.S[c * NP + j];
        }
}

}  // namespace kvar
