// api.cu -- the C ABI of libkda: argument validation, engine choice, launches.
#include <limits.h>
#include <stdarg.h>
#include <stdio.h>

#include "kda_internal.cuh"

namespace {

thread_local char g_detail[256] = "";

// Device word a kernel sets when one of its bounded waits gives up.
__device__ int g_device_error = 0;

int fail(int code, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_detail, sizeof g_detail, fmt, ap);
    va_end(ap);
    return code;
}

int cuda_fail(cudaError_t e, const char *what) {
    return fail(KDA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int *device_error_ptr() {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
    return static_cast<int *>(p);
}

struct Ptr {
    const void *p;
    const char *name;
    bool required;
};

int check_pointers(const Ptr *ps, int n) {
    for (int i = 0; i < n; ++i) {
        if (!ps[i].p) {
            if (ps[i].required) return fail(KDA_ERR_INVALID_ARG, "%s is NULL", ps[i].name);
            continue;
        }
        if (!aligned16(ps[i].p))
            return fail(KDA_ERR_ALIGNMENT, "%s is not 16-byte aligned", ps[i].name);
    }
    return KDA_OK;
}

int check_common(int dk, int dv, int dtype) {
    if (dtype != KDA_BF16 && dtype != KDA_F32)
        return fail(KDA_ERR_INVALID_ARG, "dtype %d is neither KDA_BF16 nor KDA_F32", dtype);
    if (dk < 1 || dv < 1) return fail(KDA_ERR_INVALID_ARG, "dk=%d dv=%d must be >= 1", dk, dv);
    if (dk > 128 || dv > 128)
        return fail(KDA_ERR_UNSUPPORTED, "dk=%d dv=%d: head dimensions above 128", dk, dv);
    if (dv % 4 != 0) return fail(KDA_ERR_UNSUPPORTED, "dv=%d is not a multiple of 4", dv);
    return KDA_OK;
}

}  // namespace

namespace kda {
int set_error_detail(int code, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_detail, sizeof g_detail, fmt, ap);
    va_end(ap);
    return code;
}
int *device_error_word() { return device_error_ptr(); }
}  // namespace kda

extern "C" {

int kda_version(void) { return 20000; }

const char *kda_strerror(int code) {
    switch (code) {
        case KDA_OK: return "KDA_OK";
        case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG";
        case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED";
        case KDA_ERR_ALIGNMENT: return "KDA_ERR_ALIGNMENT";
        case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE";
        case KDA_ERR_CUDA: return "KDA_ERR_CUDA";
        case KDA_ERR_DEVICE_TIMEOUT: return "KDA_ERR_DEVICE_TIMEOUT";
        default: return "KDA_ERR_UNKNOWN";
    }
}

const char *kda_last_error_detail(void) { return g_detail; }

int kda_test_inject_wait_timeout(int on) { return kda::set_test_timeout(on); }

int kda_engine_supported(int engine, int dk, int dv, int chunk, int dtype) {
    const bool generic = (dtype == KDA_BF16 || dtype == KDA_F32) && dk >= 1 && dv >= 1 &&
                         dk <= 128 && dv <= 128 && dv % 4 == 0 &&
                         (chunk == 16 || chunk == 32 || chunk == 64);
    switch (engine) {
        case KDA_ENGINE_AUTO:
        case KDA_ENGINE_GENERIC: return generic ? 1 : 0;
        case KDA_ENGINE_TC_CLUSTER:
            return generic && kda::chunk_cluster_supported(dk, dv, chunk, dtype) ? 1 : 0;
        default: return 0;
    }
}

size_t kda_workspace_bytes(int B, int T, int H, int dk, int dv, int chunk, int dtype) {
    if (B <= 0 || T <= 0 || H <= 0) return 0;
    if (kda::chunk_cluster_supported(dk, dv, chunk, dtype))
        return kda::chunk_cluster_workspace_bytes(B, H);
    return 0;
}

int kda_chunk_fwd_engine(int engine, const void *q, const void *k, const void *v,
                         const float *log_alpha, const float *beta, const float *S0, void *out,
                         float *S_T, int B, int T, int H, int dk, int dv, int chunk, int dtype,
                         void *workspace, size_t workspace_bytes, void *stream) {
    g_detail[0] = '\0';
    if (engine != KDA_ENGINE_AUTO && engine != KDA_ENGINE_GENERIC && engine != KDA_ENGINE_TC_CLUSTER)
        return fail(KDA_ERR_INVALID_ARG, "engine %d is not a kda_engine", engine);
    if (B < 0 || T < 0 || H < 0)
        return fail(KDA_ERR_INVALID_ARG, "B=%d T=%d H=%d must be >= 0", B, T, H);
    int rc = check_common(dk, dv, dtype);
    if (rc != KDA_OK) return rc;
    if (chunk != 16 && chunk != 32 && chunk != 64)
        return fail(KDA_ERR_UNSUPPORTED, "chunk=%d is not 16, 32 or 64", chunk);
    // Token rows are 32-bit tensor-map coordinates; a head is up to 4 CTAs of a 1-D grid.
    if (static_cast<long long>(B) * T > INT_MAX)
        return fail(KDA_ERR_UNSUPPORTED, "B*T = %lld tokens: more than 2^31 - 1; split the batch",
                    static_cast<long long>(B) * T);
    if (static_cast<long long>(B) * H > INT_MAX / 4)
        return fail(KDA_ERR_UNSUPPORTED, "B*H = %lld heads: more than 2^29 - 1; split the batch",
                    static_cast<long long>(B) * H);
    if (B == 0 || H == 0) return KDA_OK;
    const bool tokens = T > 0;
    const Ptr ps[] = {{q, "q", tokens},           {k, "k", tokens},       {v, "v", tokens},
                      {log_alpha, "log_alpha", tokens}, {beta, "beta", tokens}, {out, "out", tokens},
                      {S0, "S0", false},          {S_T, "S_T", false},    {workspace, "workspace", false}};
    rc = check_pointers(ps, sizeof ps / sizeof ps[0]);
    if (rc != KDA_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    if (!tokens) {  // S_T = S0 (or zeros)
        if (!S_T) return KDA_OK;
        const size_t bytes = static_cast<size_t>(B) * H * dk * dv * sizeof(float);
        cudaError_t e = S0 ? (S0 == S_T ? cudaSuccess
                                        : cudaMemcpyAsync(S_T, S0, bytes, cudaMemcpyDeviceToDevice, s))
                           : cudaMemsetAsync(S_T, 0, bytes, s);
        return e == cudaSuccess ? KDA_OK : cuda_fail(e, "copying S0 to S_T");
    }

    const bool cl_ok = kda::chunk_cluster_supported(dk, dv, chunk, dtype);
    bool use_cluster = false;
    if (engine == KDA_ENGINE_TC_CLUSTER) {
        if (!cl_ok)
            return fail(KDA_ERR_UNSUPPORTED,
                        "the tensor-core engine needs bf16, dk = dv = 128, chunk = 64 (got dtype %d, "
                        "dk %d, dv %d, chunk %d)", dtype, dk, dv, chunk);
        use_cluster = true;
    } else if (engine == KDA_ENGINE_AUTO) {
        use_cluster = cl_ok;
    }

    kda::ChunkArgs a{q, k, v, log_alpha, beta, S0, out, S_T, B, T, H, dk, dv, chunk, dtype,
                     workspace, workspace_bytes, nullptr};
    cudaError_t e;
    if (use_cluster) {
        const size_t need = kda::chunk_cluster_workspace_bytes(B, H);
        if (need > 0 && (!workspace || workspace_bytes < need))
            return fail(KDA_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed",
                        workspace ? workspace_bytes : static_cast<size_t>(0), need);
        a.device_error = device_error_ptr();
        if (!a.device_error) return fail(KDA_ERR_CUDA, "device error word not addressable");
        e = kda::launch_chunk_cluster(a, s);
    } else {
        e = kda::launch_chunk_generic(a, s);
    }
    return e == cudaSuccess ? KDA_OK : cuda_fail(e, "launching the prefill kernel");
}

namespace {
// kda_chunk_fwd_fused and kda_layer_fwd: the prefill on the tensor-core engine with the
// layer prologue, and (out_gate != NULL) the layer epilogue.
int fused_impl(const void *q, const void *k, const void *v, const void *gate, const float *beta,
               bool gated, const void *out_gate, const float *norm_weight, float eps, const float *S0, void *out,
               float *S_T, int B, int T, int H, int dk, int dv, int chunk, int dtype, void *workspace,
               size_t workspace_bytes, void *stream) {
    g_detail[0] = '\0';
    if (B < 0 || T < 0 || H < 0)
        return fail(KDA_ERR_INVALID_ARG, "B=%d T=%d H=%d must be >= 0", B, T, H);
    int rc = check_common(dk, dv, dtype);
    if (rc != KDA_OK) return rc;
    if (!kda::chunk_cluster_supported(dk, dv, chunk, dtype))
        return fail(KDA_ERR_UNSUPPORTED,
                    "the fused prologue runs on the tensor-core engine: bf16, dk = dv = 128, chunk = 64 "
                    "(got dtype %d, dk %d, dv %d, chunk %d)", dtype, dk, dv, chunk);
    if (static_cast<long long>(B) * T > INT_MAX)
        return fail(KDA_ERR_UNSUPPORTED, "B*T = %lld tokens: more than 2^31 - 1; split the batch",
                    static_cast<long long>(B) * T);
    if (static_cast<long long>(B) * H > INT_MAX / 4)
        return fail(KDA_ERR_UNSUPPORTED, "B*H = %lld heads: more than 2^29 - 1; split the batch",
                    static_cast<long long>(B) * H);
    if (B == 0 || H == 0) return KDA_OK;
    const bool tokens = T > 0;
    if (gated && !(eps >= 0.f && eps < 1e30f))
        return fail(KDA_ERR_INVALID_ARG, "eps = %g is not a finite value >= 0", static_cast<double>(eps));
    const Ptr ps[] = {{q, "q", tokens},       {k, "k", tokens},   {v, "v", tokens},
                      {gate, "gate", tokens}, {beta, "beta", tokens}, {out, "out", tokens},
                      {S0, "S0", false},      {S_T, "S_T", false}, {workspace, "workspace", false},
                      {out_gate, "out_gate", gated && tokens}, {norm_weight, "norm_weight", gated && tokens}};
    rc = check_pointers(ps, sizeof ps / sizeof ps[0]);
    if (rc != KDA_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (!tokens) {  // S_T = S0 (or zeros)
        if (!S_T) return KDA_OK;
        const size_t bytes = static_cast<size_t>(B) * H * dk * dv * sizeof(float);
        cudaError_t e = S0 ? (S0 == S_T ? cudaSuccess
                                        : cudaMemcpyAsync(S_T, S0, bytes, cudaMemcpyDeviceToDevice, s))
                           : cudaMemsetAsync(S_T, 0, bytes, s);
        return e == cudaSuccess ? KDA_OK : cuda_fail(e, "copying S0 to S_T");
    }
    const size_t need = kda::chunk_cluster_workspace_bytes(B, H);
    if (!workspace || workspace_bytes < need)
        return fail(KDA_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed",
                    workspace ? workspace_bytes : static_cast<size_t>(0), need);
    kda::ChunkArgs a{q, k, v, nullptr, beta, S0, out, S_T, B, T, H, dk, dv, chunk, dtype,
                     workspace, workspace_bytes, device_error_ptr(), gate};
    if (!a.device_error) return fail(KDA_ERR_CUDA, "device error word not addressable");
    if (gated) {
        a.out_gate = out_gate;
        a.norm_weight = norm_weight;
        a.norm_eps = eps;
    }
    const cudaError_t e = kda::launch_chunk_cluster(a, s);
    return e == cudaSuccess ? KDA_OK : cuda_fail(e, "launching the prefill kernel");
}
}  // namespace

int kda_chunk_fwd_fused(const void *q, const void *k, const void *v, const void *gate,
                        const float *beta, const float *S0, void *out, float *S_T, int B, int T,
                        int H, int dk, int dv, int chunk, int dtype, void *workspace,
                        size_t workspace_bytes, void *stream) {
    return fused_impl(q, k, v, gate, beta, false, nullptr, nullptr, 0.f, S0, out, S_T, B, T, H, dk, dv, chunk,
                      dtype, workspace, workspace_bytes, stream);
}

int kda_layer_fwd(const void *q, const void *k, const void *v, const void *gate, const float *beta,
                  const void *out_gate, const float *norm_weight, float eps, const float *S0, void *out,
                  float *S_T, int B, int T, int H, int dk, int dv, int chunk, int dtype, void *workspace,
                  size_t workspace_bytes, void *stream) {
    return fused_impl(q, k, v, gate, beta, true, out_gate, norm_weight, eps, S0, out, S_T, B, T, H, dk, dv,
                      chunk, dtype, workspace, workspace_bytes, stream);
}


int kda_chunk_fwd(const void *q, const void *k, const void *v, const float *log_alpha,
                  const float *beta, const float *S0, void *out, float *S_T, int B, int T, int H,
                  int dk, int dv, int chunk, int dtype, void *workspace, size_t workspace_bytes,
                  void *stream) {
    return kda_chunk_fwd_engine(KDA_ENGINE_AUTO, q, k, v, log_alpha, beta, S0, out, S_T, B, T, H,
                                dk, dv, chunk, dtype, workspace, workspace_bytes, stream);
}

int kda_recurrent_step(const void *q, const void *k, const void *v, const float *log_alpha,
                       const float *beta, float *state, const int32_t *slot, void *out, int N,
                       int H, int dk, int dv, int dtype, void *stream) {
    g_detail[0] = '\0';
    if (N < 0 || H < 0) return fail(KDA_ERR_INVALID_ARG, "N=%d H=%d must be >= 0", N, H);
    int rc = check_common(dk, dv, dtype);
    if (rc != KDA_OK) return rc;
    // A (sequence, head) is up to 2 CTAs of a 1-D grid.
    if (static_cast<long long>(N) * H > INT_MAX / 2)
        return fail(KDA_ERR_UNSUPPORTED, "N*H = %lld heads: more than 2^30 - 1; split the batch",
                    static_cast<long long>(N) * H);
    if (N == 0 || H == 0) return KDA_OK;
    const Ptr ps[] = {{q, "q", true},       {k, "k", true},         {v, "v", true},
                      {log_alpha, "log_alpha", true}, {beta, "beta", true}, {state, "state", true},
                      {out, "out", true},   {slot, "slot", false}};
    rc = check_pointers(ps, sizeof ps / sizeof ps[0]);
    if (rc != KDA_OK) return rc;
    kda::DecodeArgs a{q, k, v, log_alpha, beta, state, slot, out, N, H, dk, dv, dtype};
    cudaError_t e = kda::launch_decode(a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KDA_OK : cuda_fail(e, "launching the decode kernel");
}

size_t kda_bwd_workspace_bytes(int B, int T, int H, int dk, int dv, int dtype) {
    if (B <= 0 || T <= 0 || H <= 0 || dk < 1 || dv < 1 || dk > 128 || dv > 128) return 0;
    if (dtype != KDA_BF16 && dtype != KDA_F32) return 0;
    return kda::chunk_bwd_workspace_bytes(B, T, H, dk, dv);
}

int kda_chunk_bwd(const void *q, const void *k, const void *v, const float *log_alpha,
                  const float *beta, const float *S0, const void *grad_out, const float *grad_S_T,
                  void *grad_q, void *grad_k, void *grad_v, float *grad_log_alpha, float *grad_beta,
                  float *grad_S0, int B, int T, int H, int dk, int dv, int dtype, void *workspace,
                  size_t workspace_bytes, void *stream) {
    g_detail[0] = '\0';
    if (dtype != KDA_BF16 && dtype != KDA_F32)
        return fail(KDA_ERR_INVALID_ARG, "dtype %d is neither KDA_BF16 nor KDA_F32", dtype);
    if (B < 0 || T < 0 || H < 0)
        return fail(KDA_ERR_INVALID_ARG, "B=%d T=%d H=%d must be >= 0", B, T, H);
    if (dk < 1 || dv < 1) return fail(KDA_ERR_INVALID_ARG, "dk=%d dv=%d must be >= 1", dk, dv);
    if (dk > 128 || dv > 128)
        return fail(KDA_ERR_UNSUPPORTED, "dk=%d dv=%d: head dimensions above 128", dk, dv);
    if (static_cast<long long>(B) * T > INT_MAX)
        return fail(KDA_ERR_UNSUPPORTED, "B*T = %lld tokens: more than 2^31 - 1; split the batch",
                    static_cast<long long>(B) * T);
    if (static_cast<long long>(B) * H > INT_MAX / 4)
        return fail(KDA_ERR_UNSUPPORTED, "B*H = %lld heads: more than 2^29 - 1; split the batch",
                    static_cast<long long>(B) * H);
    if (B == 0 || H == 0) return KDA_OK;
    const bool tokens = T > 0;
    const Ptr ps[] = {{q, "q", tokens}, {k, "k", tokens}, {v, "v", tokens},
                      {log_alpha, "log_alpha", tokens}, {beta, "beta", tokens},
                      {grad_out, "grad_out", tokens}, {grad_q, "grad_q", tokens},
                      {grad_k, "grad_k", tokens}, {grad_v, "grad_v", tokens},
                      {grad_log_alpha, "grad_log_alpha", tokens}, {grad_beta, "grad_beta", tokens},
                      {S0, "S0", false}, {grad_S_T, "grad_S_T", false}, {grad_S0, "grad_S0", false},
                      {workspace, "workspace", false}};
    int rc = check_pointers(ps, sizeof ps / sizeof ps[0]);
    if (rc != KDA_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (!tokens) {  // grad_S0 = grad_S_T (or zeros)
        if (!grad_S0) return KDA_OK;
        const size_t bytes = static_cast<size_t>(B) * H * dk * dv * sizeof(float);
        cudaError_t e = grad_S_T ? (grad_S_T == grad_S0 ? cudaSuccess
                                                        : cudaMemcpyAsync(grad_S0, grad_S_T, bytes,
                                                                          cudaMemcpyDeviceToDevice, s))
                                 : cudaMemsetAsync(grad_S0, 0, bytes, s);
        return e == cudaSuccess ? KDA_OK : cuda_fail(e, "copying grad_S_T to grad_S0");
    }
    const size_t need = kda::chunk_bwd_workspace_bytes(B, T, H, dk, dv);
    if (!workspace || workspace_bytes < need)
        return fail(KDA_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed",
                    workspace ? workspace_bytes : static_cast<size_t>(0), need);
    cudaError_t e = kda::launch_chunk_bwd(q, k, v, log_alpha, beta, S0, grad_out, grad_S_T, grad_q,
                                          grad_k, grad_v, grad_log_alpha, grad_beta, grad_S0, B, T, H,
                                          dk, dv, dtype, workspace, s);
    return e == cudaSuccess ? KDA_OK : cuda_fail(e, "launching the backward kernels");
}

size_t kda_varlen_workspace_bytes(int N, int H, int dk, int dv, int dtype) {
    if (N <= 0 || H <= 0) return 0;
    if (kda::chunk_cluster_supported(dk, dv, 64, dtype)) return kda::chunk_cluster_workspace_bytes(N, H);
    return 0;
}

int kda_chunk_fwd_varlen(const void *q, const void *k, const void *v, const float *log_alpha,
                         const float *beta, const int32_t *cu_seqlens, const int32_t *slot,
                         const float *S0, void *out, float *S_T, int N, int total_T, int H, int dk,
                         int dv, int dtype, void *stream) {
    return kda_chunk_fwd_varlen_engine(KDA_ENGINE_GENERIC, q, k, v, log_alpha, beta, cu_seqlens, slot, S0,
                                       out, S_T, N, total_T, H, dk, dv, dtype, nullptr, 0, stream);
}

int kda_chunk_fwd_varlen_engine(int engine, const void *q, const void *k, const void *v,
                                const float *log_alpha, const float *beta, const int32_t *cu_seqlens,
                                const int32_t *slot, const float *S0, void *out, float *S_T, int N,
                                int total_T, int H, int dk, int dv, int dtype, void *workspace,
                                size_t workspace_bytes, void *stream) {
    g_detail[0] = '\0';
    if (engine != KDA_ENGINE_AUTO && engine != KDA_ENGINE_GENERIC && engine != KDA_ENGINE_TC_CLUSTER)
        return fail(KDA_ERR_INVALID_ARG, "engine %d is not a kda_engine", engine);
    if (dtype != KDA_BF16 && dtype != KDA_F32)
        return fail(KDA_ERR_INVALID_ARG, "dtype %d is neither KDA_BF16 nor KDA_F32", dtype);
    if (N < 0 || total_T < 0 || H < 0)
        return fail(KDA_ERR_INVALID_ARG, "N=%d total_T=%d H=%d must be >= 0", N, total_T, H);
    if (dk < 1 || dv < 1) return fail(KDA_ERR_INVALID_ARG, "dk=%d dv=%d must be >= 1", dk, dv);
    if (dk > 128 || dv > 128)
        return fail(KDA_ERR_UNSUPPORTED, "dk=%d dv=%d: head dimensions above 128", dk, dv);
    if (static_cast<long long>(N) * H > INT_MAX / 4)
        return fail(KDA_ERR_UNSUPPORTED, "N*H = %lld heads: more than 2^29 - 1; split the batch",
                    static_cast<long long>(N) * H);
    if (N == 0 || H == 0) return KDA_OK;
    if (!cu_seqlens) return fail(KDA_ERR_INVALID_ARG, "cu_seqlens is NULL");
    if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0)
        return fail(KDA_ERR_ALIGNMENT, "cu_seqlens is not 4-byte aligned");
    if ((reinterpret_cast<uintptr_t>(slot) & 3u) != 0)
        return fail(KDA_ERR_ALIGNMENT, "slot is not 4-byte aligned");
    const bool tokens = total_T > 0;
    const Ptr ps[] = {{q, "q", tokens}, {k, "k", tokens}, {v, "v", tokens},
                      {log_alpha, "log_alpha", tokens}, {beta, "beta", tokens}, {out, "out", tokens},
                      {S0, "S0", false}, {S_T, "S_T", false}, {workspace, "workspace", false}};
    int rc = check_pointers(ps, sizeof ps / sizeof ps[0]);
    if (rc != KDA_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the tensor-core engine: bf16, dk = dv = 128, with its operand ring in the workspace
    const bool cl_ok = kda::chunk_cluster_supported(dk, dv, 64, dtype);
    const size_t need = kda::chunk_cluster_workspace_bytes(N, H);
    bool use_cluster = false;
    if (engine == KDA_ENGINE_TC_CLUSTER) {
        if (!cl_ok)
            return fail(KDA_ERR_UNSUPPORTED,
                        "the tensor-core engine needs bf16 and dk = dv = 128 (got dtype %d, dk %d, dv %d)",
                        dtype, dk, dv);
        if (!workspace || workspace_bytes < need)
            return fail(KDA_ERR_WORKSPACE, "workspace of %zu bytes given, %zu needed",
                        workspace ? workspace_bytes : static_cast<size_t>(0), need);
        use_cluster = true;
    } else if (engine == KDA_ENGINE_AUTO) {
        use_cluster = cl_ok && workspace && workspace_bytes >= need;
    }
    cudaError_t e;
    if (use_cluster && tokens) {
        kda::ChunkArgs a{q, k, v, log_alpha, beta, S0, out, S_T, N, total_T, H, dk, dv, 64, dtype,
                         workspace, workspace_bytes, device_error_ptr()};
        if (!a.device_error) return fail(KDA_ERR_CUDA, "device error word not addressable");
        a.cu_seqlens = cu_seqlens;
        a.slot = slot;
        e = kda::launch_chunk_cluster(a, s);
    } else {   // the CUDA-core kernel (also every call without tokens: it only moves the states)
        e = kda::launch_chunk_varlen(q, k, v, log_alpha, beta, cu_seqlens, slot, S0, out, S_T, N, total_T,
                                     H, dk, dv, dtype, s);
    }
    return e == cudaSuccess ? KDA_OK : cuda_fail(e, "launching the variable-length prefill");
}

int kda_short_conv_swish(const void *x, const float *weight, const int32_t *cu_seqlens, void *y, int B,
                         int T, int H, int d, int W, int dtype, void *stream) {
    g_detail[0] = '\0';
    if (dtype != KDA_BF16 && dtype != KDA_F32)
        return fail(KDA_ERR_INVALID_ARG, "dtype %d is neither KDA_BF16 nor KDA_F32", dtype);
    if (B < 0 || T < 0 || H < 0 || d < 0)
        return fail(KDA_ERR_INVALID_ARG, "B=%d T=%d H=%d d=%d must be >= 0", B, T, H, d);
    if (W < 1 || W > 4) return fail(KDA_ERR_UNSUPPORTED, "W=%d: filters of 1..4 taps", W);
    if (d % 8 != 0) return fail(KDA_ERR_UNSUPPORTED, "d=%d is not a multiple of 8", d);
    const long long tokens = cu_seqlens ? static_cast<long long>(T) : static_cast<long long>(B) * T;
    if (tokens * H * d > (1ll << 40))
        return fail(KDA_ERR_UNSUPPORTED, "%lld x %d x %d elements: too many for one call", tokens, H, d);
    if (B == 0 || T == 0 || H == 0 || d == 0) return KDA_OK;
    if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0)
        return fail(KDA_ERR_ALIGNMENT, "cu_seqlens is not 4-byte aligned");
    const Ptr ps[] = {{x, "x", true}, {weight, "weight", true}, {y, "y", true}};
    int rc = check_pointers(ps, sizeof ps / sizeof ps[0]);
    if (rc != KDA_OK) return rc;
    if (x == y) return fail(KDA_ERR_INVALID_ARG, "y must not alias x");
    cudaError_t e = kda::launch_short_conv_swish(x, weight, y, cu_seqlens, B, T, H, d, W, dtype,
                                                 static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KDA_OK : cuda_fail(e, "launching the short convolution");
}

int kda_dplr_chunk_fwd(const void *q, const void *k, const void *v, const void *a, const void *b,
                       const float *log_alpha, const float *S0, void *out, float *S_T, int B, int T, int H,
                       int dk, int dv, int chunk, int dtype, void *stream) {
    g_detail[0] = '\0';
    if (B < 0 || T < 0 || H < 0)
        return fail(KDA_ERR_INVALID_ARG, "B=%d T=%d H=%d must be >= 0", B, T, H);
    int rc = check_common(dk, dv, dtype);
    if (rc != KDA_OK) return rc;
    if (chunk != 16 && chunk != 32) return fail(KDA_ERR_UNSUPPORTED, "chunk=%d is not 16 or 32", chunk);
    if (kda::chunk_dplr_smem_bytes(chunk, dk, dv) > 227u * 1024u)
        return fail(KDA_ERR_UNSUPPORTED, "chunk=%d with dk=%d: shared memory beyond 227 KB", chunk, dk);
    if (static_cast<long long>(B) * T > INT_MAX || static_cast<long long>(B) * H > INT_MAX / 4)
        return fail(KDA_ERR_UNSUPPORTED, "B*T = %lld, B*H = %lld: split the batch",
                    static_cast<long long>(B) * T, static_cast<long long>(B) * H);
    if (B == 0 || H == 0) return KDA_OK;
    const bool tokens = T > 0;
    const Ptr ps[] = {{q, "q", tokens}, {k, "k", tokens}, {v, "v", tokens}, {a, "a", tokens},
                      {b, "b", tokens}, {log_alpha, "log_alpha", tokens}, {out, "out", tokens},
                      {S0, "S0", false}, {S_T, "S_T", false}};
    rc = check_pointers(ps, sizeof ps / sizeof ps[0]);
    if (rc != KDA_OK) return rc;
    cudaError_t e = kda::launch_chunk_dplr(q, k, v, a, b, log_alpha, S0, out, S_T, B, T, H, dk, dv, chunk,
                                           dtype, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KDA_OK : cuda_fail(e, "launching the DPLR comparator");
}

int kda_device_status(void *stream) {
    g_detail[0] = '\0';
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "synchronising the stream");
    int flag = 0;
    e = cudaMemcpyFromSymbol(&flag, g_device_error, sizeof flag);
    if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
    if (flag == 0) return KDA_OK;
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
    return fail(KDA_ERR_DEVICE_TIMEOUT, "a bounded device wait gave up (code %d)", flag);
}

}  // extern "C"
