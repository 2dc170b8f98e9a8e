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
// (the caller forms T = X Diag(beta) from it):
//   1) X_II = (I + A_II)^{-1} for the 4 diagonal blocks: forward substitution,
//      one column per thread, fp32.
//   2) R_IJ = A_IJ X_JJ for the 6 blocks below the diagonal (one warp each); the
//      three next to the diagonal finish at once: X_{I,I-1} = -X_II R_{I,I-1}.
//   3) X_20 = -X_22 (R_20 + A_21 X_10), X_31 = -X_33 (R_31 + A_32 X_21), and the
//      first two terms of X_30's sum, R_30 + A_31 X_10.
//   4) X_30 = -X_33 (R_30 + A_31 X_10 + A_32 X_20).
// Three dependent levels of two block products each after the diagonal blocks.
// Block products use warp-level tf32 mma.sync (m16n8k8, fp32 accumulate).
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
// X_IJ = -X_II Y with Y = X's (I, J) block on entry; the result replaces Y (one warp).
template <class Out>
__device__ __forceinline__ void finish_block(float *X, int I, int J, int lane, const Out &out) {
    float r[2][4] = {};
    warp_mm16(r, blk(X, I, I), blk(X, I, J), lane);
#pragma unroll
    for (int ns = 0; ns < 2; ++ns)
#pragma unroll
        for (int e = 0; e < 4; ++e) r[ns][e] = -r[ns][e];
    __syncwarp();
    acc_store16(r, blk(X, I, J), 1.f, lane);
    acc_emit16(r, I, J, lane, out);
}

template <class Out>
__device__ inline void unit_lower_inverse(const float *A, float *X, int tid, const Out &out) {
    const int warp = tid >> 5, lane = tid & 31;
    // 1) diagonal blocks, one column per thread
    if (tid < 64) {
        const int I = tid >> 4, jj = tid & 15, base = 16 * I;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int m = 0; m < i; ++m) {
                if (m & 1) s1 = fmaf(A[(base + i) * kLD + base + m], x[m], s1);
                else s0 = fmaf(A[(base + i) * kLD + base + m], x[m], s0);
            }
            x[i] = i < jj ? 0.f : (i == jj ? 1.f : -(s0 + s1));
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            X[(base + i) * kLD + base + jj] = x[i];
            out.one(base + i, base + jj, x[i]);
        }
    }
    __syncthreads();
    // 2) warps 0..2: blocks (1,0), (2,1), (3,2), finished; warps 3..5: R_20, R_31, R_30
    if (warp < 6) {
        const int I = warp < 3 ? warp + 1 : (warp == 5 ? 3 : warp - 1);   // 1,2,3,2,3,3
        const int J = warp < 3 ? warp : (warp == 5 ? 0 : warp - 3);        // 0,1,2,0,1,0
        float acc[2][4] = {};
        warp_mm16(acc, blk(A, I, J), blk(X, J, J), lane);
        acc_store16(acc, blk(X, I, J), 1.f, lane);
        if (warp < 3) {
            __syncwarp();
            finish_block(X, I, J, lane, out);
        }
    }
    __syncthreads();
    // 3) warp 0: X_20; warp 1: X_31; warp 2: R_30 + A_31 X_10
    if (warp < 3) {
        const int I = warp == 1 ? 3 : (warp == 0 ? 2 : 3);
        const int J = warp == 1 ? 1 : 0;
        const int K = warp == 1 ? 2 : 1;   // the finished block X_KJ this step adds: A_IK X_KJ
        float acc[2][4];
        acc_load16(acc, blk(X, I, J), lane);
        warp_mm16(acc, blk(A, I, K), blk(X, K, J), lane);
        __syncwarp();
        acc_store16(acc, blk(X, I, J), 1.f, lane);
        if (warp < 2) {
            __syncwarp();
            finish_block(X, I, J, lane, out);
        }
    }
    __syncthreads();
    // 4) warp 0: X_30
    if (warp == 0) {
        float acc[2][4];
        acc_load16(acc, blk(X, 3, 0), lane);
        warp_mm16(acc, blk(A, 3, 2), blk(X, 2, 0), lane);
        __syncwarp();
        acc_store16(acc, blk(X, 3, 0), 1.f, lane);
        __syncwarp();
        finish_block(X, 3, 0, lane, out);
    }
}

}  // namespace ut
}  // namespace kda
