// ut_solve.cuh -- the UT transform of the chunked KDA form: the inverse of a
// unit lower-triangular 64x64 matrix (I + A) by forward substitution (Kimi
// Linear summary, es.news.hada.io/topic?id=31936, section "Algoritmo paralelo
// por chunks", which computes this inverse one row after another), organised
// in 16x16 blocks on the CUDA cores and warp-level tf32 tensor-core instructions.
#pragma once

#include <stdint.h>

namespace kda {
namespace ut {

constexpr int kLD = 68;  // row stride (floats) of A and X: conflict-free mma fragments

// X = (I + A)^{-1} for the strictly lower-triangular 64x64 A (row stride kLD),
// organised in 16x16 blocks, and every finished block handed to `out` as well
// (the caller forms T = X Diag(beta) from it). With N_IJ = X_II A_IJ, block
// forward substitution reads X_IJ = -sum_{J<=K<I} N_IK X_KJ:
//   1) X_II = (I + A_II)^{-1} for the 4 diagonal blocks, one column per thread,
//      fp32, in 8x8 halves (forward substitution inside each half, then the
//      lower-left half as -X_11 A_10 X_00).
//   2) one warp per block below the diagonal: N_IJ (kept in A's (I,J) block),
//      then -N_IJ X_JJ, which is X_IJ itself next to the diagonal (J = I-1)
//      and the first term of X_20, X_31, X_30 otherwise.
//   3) X_20 -= N_21 X_10, X_31 -= N_32 X_21, X_30 -= N_31 X_10.
//   4) X_30 -= N_32 X_20.
// Four dependent block products after the diagonal blocks. Block products use
// warp-level tf32 mma.sync (m16n8k8, fp32 accumulate). The solve overwrites
// A's blocks below the diagonal.
// `out.one(i, j, x)` receives single elements of the diagonal blocks (all of
// them, zeros above the diagonal included); `out.pair(i, j, x0, x1)` receives
// elements (i, j), (i, j + 1) of the blocks below the diagonal, j even.

__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

// acc[ns][.] += A(16x16) * B(16x16) for one warp; acc holds the two 16x8 halves
// of the 16x16 result in the m16n8 accumulator layout.
__device__ __forceinline__ void warp_mm16(float (&acc)[2][4], const float *A, const float *B,
                                          int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        uint32_t a[4];
        a[0] = to_tf32(A[g * kLD + 8 * ks + t]);
        a[1] = to_tf32(A[(g + 8) * kLD + 8 * ks + t]);
        a[2] = to_tf32(A[g * kLD + 8 * ks + t + 4]);
        a[3] = to_tf32(A[(g + 8) * kLD + 8 * ks + t + 4]);
#pragma unroll
        for (int ns = 0; ns < 2; ++ns) {
            const uint32_t b0 = to_tf32(B[(8 * ks + t) * kLD + 8 * ns + g]);
            const uint32_t b1 = to_tf32(B[(8 * ks + t + 4) * kLD + 8 * ns + g]);
            asm volatile(
                "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
                "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                : "+f"(acc[ns][0]), "+f"(acc[ns][1]), "+f"(acc[ns][2]), "+f"(acc[ns][3])
                : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
        }
    }
}
__device__ __forceinline__ void acc_load16(float (&acc)[2][4], const float *C, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int ns = 0; ns < 2; ++ns) {
        acc[ns][0] = C[g * kLD + 8 * ns + 2 * t];
        acc[ns][1] = C[g * kLD + 8 * ns + 2 * t + 1];
        acc[ns][2] = C[(g + 8) * kLD + 8 * ns + 2 * t];
        acc[ns][3] = C[(g + 8) * kLD + 8 * ns + 2 * t + 1];
    }
}
__device__ __forceinline__ void acc_store16(const float (&acc)[2][4], float *C, float scale,
                                            int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int ns = 0; ns < 2; ++ns) {
        C[g * kLD + 8 * ns + 2 * t] = scale * acc[ns][0];
        C[g * kLD + 8 * ns + 2 * t + 1] = scale * acc[ns][1];
        C[(g + 8) * kLD + 8 * ns + 2 * t] = scale * acc[ns][2];
        C[(g + 8) * kLD + 8 * ns + 2 * t + 1] = scale * acc[ns][3];
    }
}
__device__ __forceinline__ const float *blk(const float *M, int I, int J) {
    return M + 16 * I * kLD + 16 * J;
}
__device__ __forceinline__ float *blk(float *M, int I, int J) { return M + 16 * I * kLD + 16 * J; }

template <class Out>
__device__ __forceinline__ void acc_emit16(const float (&acc)[2][4], int I, int J, int lane, const Out &out) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int ns = 0; ns < 2; ++ns) {
        out.pair(16 * I + g, 16 * J + 8 * ns + 2 * t, acc[ns][0], acc[ns][1]);
        out.pair(16 * I + g + 8, 16 * J + 8 * ns + 2 * t, acc[ns][2], acc[ns][3]);
    }
}
template <class Out>
__device__ inline void unit_lower_inverse(float *A, float *X, int tid, const Out &out) {
    const int warp = tid >> 5, lane = tid & 31;
    // 1) diagonal blocks, one column per thread, each in 8x8 halves: the column's own
    //    8x8 diagonal sub-block by forward substitution, then (columns 0..7) the rows
    //    below it as -X_11 (A_10 x) with the neighbour columns' X_11 from shared memory
    if (tid < 64) {
        const int I = tid >> 4, jj = tid & 15, base = 16 * I, lo = jj & 8;
        const float *Ab = A + base * kLD + base;
        float *Xb = X + base * kLD + base;
        float xa[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const int i = lo + r;
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int m = 0; m < r; ++m) {
                const float a = Ab[i * kLD + lo + m];
                if (m & 1) s1 = fmaf(a, xa[m], s1);
                else s0 = fmaf(a, xa[m], s0);
            }
            xa[r] = i < jj ? 0.f : (i == jj ? 1.f : -(s0 + s1));
        }
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            Xb[(lo + r) * kLD + jj] = xa[r];
            out.one(base + lo + r, base + jj, xa[r]);
        }
        __syncwarp();
        if (jj < 8) {
            float y[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                float s0 = 0.f, s1 = 0.f;
#pragma unroll
                for (int m = 0; m < 8; m += 2) {
                    s0 = fmaf(Ab[(8 + r) * kLD + m], xa[m], s0);
                    s1 = fmaf(Ab[(8 + r) * kLD + m + 1], xa[m + 1], s1);
                }
                y[r] = s0 + s1;
            }
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                float z = 0.f;
#pragma unroll
                for (int m = 0; m <= r; ++m) z = fmaf(Xb[(8 + r) * kLD + 8 + m], y[m], z);
                Xb[(8 + r) * kLD + jj] = -z;
                out.one(base + 8 + r, base + jj, -z);
            }
        } else {
#pragma unroll
            for (int r = 0; r < 8; ++r) {   // rows 0..7 of columns 8..15
                Xb[r * kLD + jj] = 0.f;
                out.one(base + r, base + jj, 0.f);
            }
        }
    }
    __syncthreads();
    // 2) warps 0..5 take blocks (1,0), (2,1), (3,2), (2,0), (3,1), (3,0)
    if (warp < 6) {
        const int I = warp < 3 ? warp + 1 : (warp == 5 ? 3 : warp - 1);
        const int J = warp < 3 ? warp : (warp == 5 ? 0 : warp - 3);
        float n[2][4] = {};
        warp_mm16(n, blk(X, I, I), blk(A, I, J), lane);   // N_IJ = X_II A_IJ
        __syncwarp();
        acc_store16(n, blk(A, I, J), 1.f, lane);
        __syncwarp();
        float y[2][4] = {};
        warp_mm16(y, blk(A, I, J), blk(X, J, J), lane);   // N_IJ X_JJ
        acc_store16(y, blk(X, I, J), -1.f, lane);
        if (warp < 3) {
#pragma unroll
            for (int ns = 0; ns < 2; ++ns)
#pragma unroll
                for (int e = 0; e < 4; ++e) y[ns][e] = -y[ns][e];
            acc_emit16(y, I, J, lane, out);
        }
    }
    __syncthreads();
    // 3) warp 0: X_20 -= N_21 X_10; warp 1: X_31 -= N_32 X_21; warp 2: X_30 -= N_31 X_10
    if (warp < 3) {
        const int I = warp == 0 ? 2 : 3, J = warp == 1 ? 1 : 0, K = warp == 1 ? 2 : 1;
        float acc[2][4], t[2][4] = {};
        acc_load16(acc, blk(X, I, J), lane);
        warp_mm16(t, blk(A, I, K), blk(X, K, J), lane);
#pragma unroll
        for (int ns = 0; ns < 2; ++ns)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[ns][e] -= t[ns][e];
        acc_store16(acc, blk(X, I, J), 1.f, lane);
        if (warp < 2) acc_emit16(acc, I, J, lane, out);
    }
    __syncthreads();
    // 4) warp 0: X_30 -= N_32 X_20
    if (warp == 0) {
        float acc[2][4], t[2][4] = {};
        acc_load16(acc, blk(X, 3, 0), lane);
        warp_mm16(t, blk(A, 3, 2), blk(X, 2, 0), lane);
#pragma unroll
        for (int ns = 0; ns < 2; ++ns)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[ns][e] -= t[ns][e];
        acc_store16(acc, blk(X, 3, 0), 1.f, lane);
        acc_emit16(acc, 3, 0, lane, out);
    }
}

}  // namespace ut
}  // namespace kda
