// kda_internal.cuh -- declarations shared by the libkda translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kda.h"

namespace kda {

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

struct ChunkArgs {
    const void *q, *k, *v;
    const float *log_alpha, *beta, *S0;
    void *out;
    float *S_T;
    int B, T, H, dk, dv, chunk, dtype;
    void *workspace;
    size_t workspace_bytes;
    int *device_error;  // set to a nonzero code by a kernel whose bounded wait gave up
    const void *gate = nullptr;  // fused layer prologue: gate pre-activation (log_alpha unused)
    // packed sequences: B = N sequences, T = the packed total; sequence n is tokens
    // cu_seqlens[n] .. cu_seqlens[n+1]-1 and uses state row slot[n] (n without a slot map)
    const int32_t *cu_seqlens = nullptr;
    const int32_t *slot = nullptr;
    // layer epilogue (with the fused prologue): out = RMSNorm(o) * norm_weight * sigmoid(out_gate)
    const void *out_gate = nullptr;
    const float *norm_weight = nullptr;
    float norm_eps = 1e-6f;
    // the workspace's ring pool is this library's fixed array: its in-use bitmap is kept
    // clear between calls rather than cleared by each launch
    bool fixed_pool = false;
};

struct DecodeArgs {
    const void *q, *k, *v;
    const float *log_alpha, *beta;
    float *state;
    const int32_t *slot;
    void *out;
    int N, H, dk, dv, dtype;
};

// Launchers return cudaSuccess or the launch error. They do no argument checks.
cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s);
cudaError_t launch_chunk_generic(const ChunkArgs &a, cudaStream_t s);
cudaError_t launch_chunk_cluster(const ChunkArgs &a, cudaStream_t s);

// Records `fmt` as the calling thread's kda_last_error_detail() and returns code.
int set_error_detail(int code, const char *fmt, ...);
// Device address of the word kernels set when a bounded wait gives up (nullptr on error).
int *device_error_word();

bool chunk_cluster_supported(int dk, int dv, int chunk, int dtype);
// Test hook of the cluster engine's give-up path (kda_test_inject_wait_timeout); returns the old value.
int set_test_timeout(int on);
size_t chunk_cluster_workspace_bytes(int B, int H);
// Backward pass (chunk_bwd.cu).
size_t chunk_bwd_workspace_bytes(int B, int T, int H, int dk, int dv);
cudaError_t launch_chunk_bwd(const void *q, const void *k, const void *v, const float *la,
                             const float *beta, const float *S0, const void *dout, const float *dS_T,
                             void *dq, void *dk_, void *dv_, float *dla, float *dbeta, float *dS0, int B,
                             int T, int H, int dk, int dv, int dtype, void *ws, cudaStream_t s);
// Variable-length prefill (chunk_varlen.cu).
cudaError_t launch_chunk_varlen(const void *q, const void *k, const void *v, const float *la,
                                const float *beta, const int32_t *cu_seqlens, const int32_t *slot,
                                const float *S0, void *out, float *S_T, int N, int total_T, int H,
                                int dk, int dv, int dtype, cudaStream_t s);
// ShortConv + Swish (short_conv.cu): dense [B,T,H,d], or B packed sequences over T tokens.
cudaError_t launch_short_conv_swish(const void *x, const float *w, void *y, const int32_t *cu_seqlens,
                                    int B, int T, int H, int d, int W, int dtype, cudaStream_t s);
// General DPLR comparator (chunk_dplr.cu).
size_t chunk_dplr_smem_bytes(int chunk, int dk, int dv);
cudaError_t launch_chunk_dplr(const void *q, const void *k, const void *v, const void *a, const void *b,
                              const float *la, const float *S0, void *out, float *S_T, int B, int T, int H,
                              int dk, int dv, int chunk, int dtype, cudaStream_t s);
// Ring of operand images of the cluster engine: 3 producers x 3 slots of 81 KB. A workspace
// holds a pool of rings behind a 256-byte in-use bitmap; each 4-CTA cluster (one sequence
// and head) claims a ring when it starts and releases it when it ends, so the pool needs
// only as many rings as clusters can be resident at once (148 SMs / 4 = 37 on B200).
constexpr size_t kClusterRingBytesPerHead = 9ull * 82944;
constexpr int kClusterMaxRings = 40;
constexpr size_t kClusterPoolHeader = 256;

}  // namespace kda
