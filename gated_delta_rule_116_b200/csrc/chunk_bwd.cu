// chunk_bwd.cu -- kernels and launch of the chunked KDA backward (bodies in
// chunk_bwd.cuh). Workspace: the entry state of every chunk (fp32
// [B,H,chunks,dk,dv]) and fp32 accumulators for dq and dk, cast to the input
// dtype at the end.
#include "kda_internal.cuh"
#include "tc_sm100.cuh"

namespace kda {
#include "chunk_bwd.cuh"
namespace {

template <typename Tin>
__global__ void __launch_bounds__(kbwd::kThreads, 1)
bwd_states_kernel(const Tin *q, const Tin *k, const Tin *v, const float *la, const float *beta,
                  const float *S0, float *states, int T, int H, int dk, int dv) {
    extern __shared__ float sm[];
    kbwd::states_body<Tin>(sm, q, k, v, la, beta, S0, states, T, H, dk, dv);
}

template <typename Tin>
__global__ void __launch_bounds__(kbwd::kThreads, 1)
bwd_chunk_kernel(const Tin *q, const Tin *k, const Tin *v, const float *la, const float *beta,
                 const Tin *dout, const float *dS_T, const float *states, float *dq_acc,
                 float *dk_acc, Tin *dv_out, float *dla, float *dbeta, float *dS0, int T, int H,
                 int dk, int dv) {
    extern __shared__ float sm[];
    kbwd::bwd_body<Tin>(sm, q, k, v, la, beta, dout, dS_T, states, dq_acc, dk_acc, dv_out, dla,
                        dbeta, dS0, T, H, dk, dv);
}

template <typename Tout>
__global__ void cast_kernel(const float *src, Tout *dst, long n) {
    for (long i = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<long>(gridDim.x) * blockDim.x)
        dst[i] = from_f32<Tout>(src[i]);
}

template <typename Tin>
cudaError_t launch_typed(const void *q, const void *k, const void *v, const float *la,
                         const float *beta, const float *S0, const void *dout, const float *dS_T,
                         void *dq, void *dk_, void *dv_, float *dla, float *dbeta, float *dS0, int B,
                         int T, int H, int dk, int dv, float *ws, cudaStream_t s) {
    const kbwd::Layout L(dk, kbwd::kNV);
    const size_t smem = L.floats() * sizeof(float);
    const long nk = static_cast<long>(B) * T * H * dk;
    const int nchunks = (T + kbwd::kC - 1) / kbwd::kC;
    float *states = ws;
    float *dq_acc = states + static_cast<long>(B) * H * nchunks * dk * dv;
    float *dk_acc = dq_acc + nk;
    cudaError_t e;
    if ((e = cudaMemsetAsync(dq_acc, 0, 2 * nk * sizeof(float), s)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dla, 0, nk * sizeof(float), s)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dbeta, 0, static_cast<long>(B) * T * H * sizeof(float), s)) != cudaSuccess) return e;
    auto ks = bwd_states_kernel<Tin>;
    auto kb = bwd_chunk_kernel<Tin>;
    if ((e = cudaFuncSetAttribute(ks, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem))) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(kb, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem))) != cudaSuccess) return e;
    const dim3 grid(static_cast<unsigned>(B) * H, (dv + kbwd::kNV - 1) / kbwd::kNV);
    ks<<<grid, kbwd::kThreads, smem, s>>>(static_cast<const Tin *>(q), static_cast<const Tin *>(k),
                                          static_cast<const Tin *>(v), la, beta, S0, states, T, H, dk, dv);
    kb<<<grid, kbwd::kThreads, smem, s>>>(static_cast<const Tin *>(q), static_cast<const Tin *>(k),
                                          static_cast<const Tin *>(v), la, beta,
                                          static_cast<const Tin *>(dout), dS_T, states, dq_acc, dk_acc,
                                          static_cast<Tin *>(dv_), dla, dbeta, dS0, T, H, dk, dv);
    cast_kernel<Tin><<<592, 256, 0, s>>>(dq_acc, static_cast<Tin *>(dq), nk);
    cast_kernel<Tin><<<592, 256, 0, s>>>(dk_acc, static_cast<Tin *>(dk_), nk);
    return cudaGetLastError();
}

}  // namespace

size_t chunk_bwd_workspace_bytes(int B, int T, int H, int dk, int dv) {
    const long nchunks = (T + kbwd::kC - 1) / kbwd::kC;
    return (static_cast<size_t>(B) * H * nchunks * dk * dv + 2ull * B * T * H * dk) * sizeof(float);
}

cudaError_t launch_chunk_bwd(const void *q, const void *k, const void *v, const float *la,
                             const float *beta, const float *S0, const void *dout, const float *dS_T,
                             void *dq, void *dk_, void *dv_, float *dla, float *dbeta, float *dS0, int B,
                             int T, int H, int dk, int dv, int dtype, void *ws, cudaStream_t s) {
    return dtype == KDA_BF16
               ? launch_typed<__nv_bfloat16>(q, k, v, la, beta, S0, dout, dS_T, dq, dk_, dv_, dla, dbeta,
                                             dS0, B, T, H, dk, dv, static_cast<float *>(ws), s)
               : launch_typed<float>(q, k, v, la, beta, S0, dout, dS_T, dq, dk_, dv_, dla, dbeta, dS0,
                                     B, T, H, dk, dv, static_cast<float *>(ws), s);
}

}  // namespace kda
