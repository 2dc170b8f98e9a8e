// chunk_static.cu -- kda_chunk_fwd_static: the cluster prefill engine with its
// scratch in a fixed device array of this library, for callers that cannot
// allocate device memory when they call us.
//
// Who cannot allocate: a serving process that hands all free device memory to
// its own cache/pool allocator at start-up (a cudaMalloc from inside a library
// then fails or fragments that pool); a plug-in running inside a host
// framework that owns every allocation; code on a path where an allocation
// would synchronise the device or is simply not allowed. Such callers pass
// only inputs and outputs here. The scratch the engine needs -- the pool of
// rings of per-chunk operand images its producer CTAs hand to the state-chain
// CTA -- lives in g_static_ring below: kClusterMaxRings rings behind an in-use
// bitmap, which every cluster (one sequence and head) claims a ring from when it
// starts and returns it to when it ends, so any number of heads fits.
//
// Properties a caller has to know:
//  * every GPU that loads this library holds kStaticBytes (29.9 MiB) of device
//    memory for the array until the process exits;
//  * the first call on each device looks up the array's device address
//    (cudaGetSymbolAddress, with that device current); make that first call
//    before any stream capture;
//  * the bitmap starts clear (the array is zero when the module loads) and every
//    call leaves it clear; the rings keep the last call's contents, and no ring
//    needs to start at zero (each chunk's image is written before it is read).
//    Calls that overlap on the GPU (other streams, other threads) claim
//    different rings, so they may overlap;
//  * nothing here allocates: no cudaMalloc, no cudaFree, no library routine
//    that allocates.
#include <cuda.h>
#include <limits.h>
#include <stdarg.h>
#include <stdio.h>

#include <mutex>

#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr size_t kStaticBytes = kClusterPoolHeader + kClusterMaxRings * kClusterRingBytesPerHead;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_static_ring[kStaticBytes];

std::mutex g_setup_mutex;
// Device address of g_static_ring per device, and the context it was looked up
// in: after a device reset (or a released and re-created primary context) the
// module is loaded again and the address must be looked up again.
void *g_ring_address[kMaxDevices];
CUcontext g_ring_context[kMaxDevices];

// cuCtxGetCurrent through the runtime's driver entry point (the library does not
// link the driver library directly, so it still loads where no driver exists).
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
CUcontext current_context() {
    static CtxGetCurrentFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &qr) != cudaSuccess ||
            qr != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<CtxGetCurrentFn>(p);
    }
    CUcontext ctx = nullptr;
    return fn(&ctx) == CUDA_SUCCESS ? ctx : nullptr;
}

// Device address of the array on the current device, looked up once per device
// and context. cudaGetSymbolAddress makes the device's primary context current
// on its first use, so the context is read again after it.
cudaError_t ring_address(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    CUcontext ctx = current_context();
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!ctx || !g_ring_address[dev] || g_ring_context[dev] != ctx) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_ring);
        if (e != cudaSuccess) return e;
        ctx = current_context();
        if (!ctx) return cudaErrorDeviceUninitialized;
        g_ring_address[dev] = p;
        g_ring_context[dev] = ctx;
    }
    *out = g_ring_address[dev];
    return cudaSuccess;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace kda

extern "C" int kda_chunk_fwd_static(const void *q, const void *k, const void *v,
                                    const float *log_alpha, const float *beta, const float *S0,
                                    void *out, float *S_T, int B, int T, int H, int dk, int dv,
                                    int chunk, int dtype, void *stream) {
    using namespace kda;
    if (B < 0 || T < 0 || H < 0)
        return set_error_detail(KDA_ERR_INVALID_ARG, "B=%d T=%d H=%d must be >= 0", B, T, H);
    if (dtype != KDA_BF16 || dk != 128 || dv != 128 || chunk != 64)
        return set_error_detail(KDA_ERR_UNSUPPORTED,
                                "kda_chunk_fwd_static runs the cluster engine only: bf16, "
                                "dk = dv = 128, chunk = 64 (got dtype %d, dk %d, dv %d, chunk %d)",
                                dtype, dk, dv, chunk);
    // Token rows are 32-bit tensor-map coordinates, as in kda_chunk_fwd.
    if (static_cast<long long>(B) * T > INT_MAX)
        return set_error_detail(KDA_ERR_UNSUPPORTED,
                                "B*T = %lld tokens: more than 2^31 - 1; split the batch",
                                static_cast<long long>(B) * T);
    if (static_cast<long long>(B) * H > INT_MAX / 4)
        return set_error_detail(KDA_ERR_UNSUPPORTED, "B*H = %lld heads: more than 2^29 - 1; split the batch",
                                static_cast<long long>(B) * H);
    if (chunk_cluster_workspace_bytes(B, H) > kStaticBytes)
        return set_error_detail(KDA_ERR_UNSUPPORTED, "fixed scratch too small for this problem");
    if (B == 0 || H == 0) return set_error_detail(KDA_OK, "");
    const bool tokens = T > 0;
    const void *ptrs[] = {q, k, v, log_alpha, beta, out};
    const char *names[] = {"q", "k", "v", "log_alpha", "beta", "out"};
    for (int i = 0; i < 6; ++i) {
        if (!ptrs[i] && tokens) return set_error_detail(KDA_ERR_INVALID_ARG, "%s is NULL", names[i]);
        if (ptrs[i] && !aligned16(ptrs[i]))
            return set_error_detail(KDA_ERR_ALIGNMENT, "%s is not 16-byte aligned", names[i]);
    }
    if ((S0 && !aligned16(S0)) || (S_T && !aligned16(S_T)))
        return set_error_detail(KDA_ERR_ALIGNMENT, "S0/S_T is not 16-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (!tokens) {  // S_T = S0 (or zeros)
        if (!S_T) return set_error_detail(KDA_OK, "");
        const size_t bytes = static_cast<size_t>(B) * H * dk * dv * sizeof(float);
        cudaError_t e = S0 ? (S0 == S_T ? cudaSuccess
                                        : cudaMemcpyAsync(S_T, S0, bytes, cudaMemcpyDeviceToDevice, s))
                           : cudaMemsetAsync(S_T, 0, bytes, s);
        return e == cudaSuccess ? set_error_detail(KDA_OK, "")
                                : set_error_detail(KDA_ERR_CUDA, "copying S0 to S_T: %s",
                                                   cudaGetErrorString(e));
    }
    void *ring = nullptr;
    cudaError_t e = ring_address(&ring);
    if (e != cudaSuccess)
        return set_error_detail(KDA_ERR_CUDA, "looking up the fixed scratch: %s", cudaGetErrorString(e));
    int *err_word = device_error_word();
    if (!err_word) return set_error_detail(KDA_ERR_CUDA, "device error word not addressable");
    ChunkArgs a{q, k, v, log_alpha, beta, S0, out, S_T, B, T, H, dk, dv, chunk, dtype,
                ring, kStaticBytes, err_word};
    a.fixed_pool = true;
    e = launch_chunk_cluster(a, s);
    return e == cudaSuccess ? set_error_detail(KDA_OK, "")
                            : set_error_detail(KDA_ERR_CUDA, "launching the prefill kernel: %s",
                                               cudaGetErrorString(e));
}
