// chunk_varlen.cu -- kernel and launch of the variable-length prefill (body in
// chunk_varlen.cuh, chunk terms shared with the backward pass in chunk_bwd.cuh).
#include "kda_internal.cuh"
#include "tc_sm100.cuh"

namespace kda {
#include "chunk_bwd.cuh"
#include "chunk_varlen.cuh"
namespace {

template <typename Tin>
__global__ void __launch_bounds__(kbwd::kThreads, 1)
varlen_kernel(const Tin *q, const Tin *k, const Tin *v, const float *la, const float *beta,
              const int32_t *cu_seqlens, const int32_t *slot, const float *S0, Tin *out, float *S_T,
              int total_T, int H, int dk, int dv) {
    extern __shared__ float sm[];
    kvar::varlen_body<Tin>(sm, q, k, v, la, beta, cu_seqlens, slot, S0, out, S_T, total_T, H, dk, dv);
}

template <typename Tin>
cudaError_t launch_typed(const void *q, const void *k, const void *v, const float *la,
                         const float *beta, const int32_t *cu_seqlens, const int32_t *slot,
                         const float *S0, void *out, float *S_T, int N, int total_T, int H, int dk,
                         int dv, cudaStream_t s) {
    const kbwd::Layout L(dk, kbwd::kNV);
    const size_t smem = L.floats() * sizeof(float);
    auto kern = varlen_kernel<Tin>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const dim3 grid(static_cast<unsigned>(N) * H, (dv + kbwd::kNV - 1) / kbwd::kNV);
    kern<<<grid, kbwd::kThreads, smem, s>>>(static_cast<const Tin *>(q), static_cast<const Tin *>(k),
                                            static_cast<const Tin *>(v), la, beta, cu_seqlens, slot, S0,
                                            static_cast<Tin *>(out), S_T, total_T, H, dk, dv);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_varlen(const void *q, const void *k, const void *v, const float *la,
                                const float *beta, const int32_t *cu_seqlens, const int32_t *slot,
                                const float *S0, void *out, float *S_T, int N, int total_T, int H,
                                int dk, int dv, int dtype, cudaStream_t s) {
    return dtype == KDA_BF16
               ? launch_typed<__nv_bfloat16>(q, k, v, la, beta, cu_seqlens, slot, S0, out, S_T, N,
                                             total_T, H, dk, dv, s)
               : launch_typed<float>(q, k, v, la, beta, cu_seqlens, slot, S0, out, S_T, N, total_T,
                                     H, dk, dv, s);
}

}  // namespace kda
