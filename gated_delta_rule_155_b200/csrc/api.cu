// api.cu — the C ABI of libkda.so (declared in include/kda.h).
//
// Every entry point validates all of its arguments before launching anything, so an
// error status means nothing ran and no output was touched.  The library allocates no
// device memory per call.  Its state: one device error word per GPU (set by a kernel
// whose bounded wait gave up), the process-wide wait limit and failure injection of
// kda_set_wait_test_hooks, and the KDA_NOALLOC_SCRATCH_BYTES array of noalloc.cu, which
// every GPU that loads the library holds until exit.
#include <algorithm>
#include <atomic>
#include <cstdint>
#include <mutex>

#include "../../include/kda.h"
#include "common.cuh"
#include "internal.h"

namespace {

__device__ int g_kda_error_word;

constexpr int kMaxDevices = 64;
std::once_flag g_err_once[kMaxDevices];
int *g_err_ptr[kMaxDevices];

// Device address of the error word on the current device (nullptr if unavailable).
int *error_word()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::call_once(g_err_once[dev], [dev] {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_kda_error_word) == cudaSuccess) g_err_ptr[dev] = (int *)p;
        else cudaGetLastError();
    });
    return g_err_ptr[dev];
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }
bool head_dim_ok(int d) { return d == 64 || d == 128; }

kda_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA; }

kda::IoType io_of(kda_dtype_t io) { return io == KDA_BF16 ? kda::IO_BF16 : kda::IO_F32; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct LayerWorkspace {
    size_t q, k, v, g, beta, o, total;
};

LayerWorkspace layer_workspace(int B, int T, int H, int dk, int dv)
{
    const size_t n = (size_t)B * T * H;
    LayerWorkspace w{};
    size_t off = 0;
    w.q = off; off = round_up(off + n * dk * sizeof(float), 256);
    w.k = off; off = round_up(off + n * dk * sizeof(float), 256);
    w.v = off; off = round_up(off + n * dv * sizeof(float), 256);
    w.g = off; off = round_up(off + n * dk * sizeof(float), 256);
    w.beta = off; off = round_up(off + n * sizeof(float), 256);
    w.o = off; off = round_up(off + n * dv * sizeof(float), 256);
    w.total = off;
    return w;
}

// The layer core runs as one tensor-core kernel (no workspace) for bf16 at dk = dv = 128;
// other dtypes and head dims run prologue -> exact fp32 chunk kernel -> epilogue.
bool layer_on_tensor_cores(kda_dtype_t io, int dk, int dv) { return io == KDA_BF16 && dk == 128 && dv == 128; }

// Shapes common to every entry point.
kda_status_t check_dims(int B, int T, int H, int dk, int dv, kda_dtype_t io)
{
    if (B < 1 || H < 1 || T < 0) return KDA_ERR_INVALID_ARG;
    if (io != KDA_F32 && io != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (!head_dim_ok(dk) || !head_dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    // index arithmetic uses 32-bit token counts and 64-bit element offsets
    if ((long long)B * T > INT32_MAX / 2 || (long long)B * H > INT32_MAX / 2) return KDA_ERR_UNSUPPORTED;
    if ((long long)B * T * H > INT32_MAX / 2) return KDA_ERR_UNSUPPORTED;
    return KDA_OK;
}

// One kernel per (dtype, head dims): bf16 at dk = dv = 128 runs on the tensor cores and
// nowhere else — a device or driver that cannot run that kernel gets KDA_ERR_UNSUPPORTED,
// not a slower kernel; fp32 at d = 128 runs the exact fp32 kernel; the other head-dim
// pairs run the exact CUDA-core kernel.
kda_status_t launch_chunked(const kda::ChunkArgs &a, cudaStream_t s)
{
    if (a.io == kda::IO_BF16 && a.dk == 128 && a.dv == 128) {
        if (!kda::chunk_tc_supported(a)) return KDA_ERR_UNSUPPORTED;
        return cuda_status(kda::launch_chunk_tc(a, s));
    }
    if (kda::chunk_f32_supported(a)) return cuda_status(kda::launch_chunk_f32(a, s));
    return cuda_status(kda::launch_chunk_simt(a, s));
}

// The layer core for B sequences of T tokens, or (cu != nullptr) for B packed sequences
// with offsets cu over a token axis of T rows; dims already checked.
kda_status_t layer_core(const void *q_raw, const void *k_raw, const void *v_raw, const float *conv_q,
                        const float *conv_k, const float *conv_v, const void *g_raw, const float *A_log,
                        const float *dt_bias, float gate_lower_bound, const void *b_raw, const void *o_gate_raw,
                        const float *o_norm_w, float norm_eps, const float *initial_state, void *out,
                        float *final_state, void *workspace, size_t workspace_bytes, int B, int T, int H, int dk,
                        int dv, kda_dtype_t io, kda_stream_t stream, const int *cu)
{
    if (!(norm_eps >= 0.0f) || !(gate_lower_bound <= 0.0f)) return KDA_ERR_INVALID_ARG;
    if (T > 0 && (!q_raw || !k_raw || !v_raw || !conv_q || !conv_k || !conv_v || !g_raw ||
                  !A_log || !b_raw || !o_gate_raw || !out))
        return KDA_ERR_INVALID_ARG;
    const void *ptrs[] = {q_raw, k_raw, v_raw, conv_q, conv_k, conv_v, g_raw, A_log, dt_bias,
                          b_raw, o_gate_raw, o_norm_w, initial_state, out, final_state};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_MISALIGNED;
    cudaStream_t s = (cudaStream_t)stream;
    if (T == 0) return cuda_status(kda::launch_fill_state(initial_state, final_state,
                                                          (size_t)B * H * dk * dv, s));
    if (layer_on_tensor_cores(io, dk, dv)) {
        // one tcgen05 kernel for the whole layer core, no workspace; where it cannot run the call
        // is refused rather than given to a slower kernel
        if (((uintptr_t)b_raw & 3) != 0) return KDA_ERR_MISALIGNED;
        kda::LayerTcArgs la{q_raw, k_raw, v_raw, g_raw, b_raw, o_gate_raw, conv_q, conv_k, conv_v, A_log,
                            dt_bias, o_norm_w, gate_lower_bound, norm_eps, initial_state, final_state, out,
                            B, T, H, dk, dv, kda::IO_BF16, error_word(), cu};
        if (!kda::layer_tc_supported(la)) return KDA_ERR_UNSUPPORTED;
        return cuda_status(kda::launch_layer_tc(la, s));
    }
    const int rows = cu ? 1 : B;   // batch rows of the token-major tensors
    const LayerWorkspace w = layer_workspace(rows, T, H, dk, dv);
    if (!workspace || workspace_bytes < w.total) return KDA_ERR_WORKSPACE;
    if (((uintptr_t)workspace & 255u) != 0) return KDA_ERR_MISALIGNED;
    char *ws = (char *)workspace;
    float *wq = (float *)(ws + w.q), *wk = (float *)(ws + w.k), *wv = (float *)(ws + w.v);
    float *wg = (float *)(ws + w.g), *wb = (float *)(ws + w.beta), *wo = (float *)(ws + w.o);

    kda::PrologueArgs pa{q_raw, k_raw, v_raw, g_raw, b_raw, conv_q, conv_k, conv_v, A_log, dt_bias,
                         gate_lower_bound, wq, wk, wv, wg, wb, rows, T, H, dk, dv, io_of(io), cu, cu ? B : 0};
    cudaError_t e = kda::launch_prologue(pa, s);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    kda::ChunkArgs ca{wq, wk, wv, wg, wb, initial_state, wo, final_state, B, T, H, dk, dv,
                      kda::IO_F32, true, true, true, true, error_word(), cu};
    e = kda::chunk_f32_supported(ca) ? kda::launch_chunk_f32(ca, s) : kda::launch_chunk_simt(ca, s);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    kda::EpilogueArgs ea{wo, o_gate_raw, o_norm_w, norm_eps, out, rows, T, H, dv, io_of(io)};
    return cuda_status(kda::launch_epilogue(ea, s));
}

}  // namespace

extern "C" {

const char *kda_status_string(kda_status_t s)
{
    switch (s) {
    case KDA_OK: return "ok";
    case KDA_ERR_INVALID_ARG: return "invalid argument (null pointer, non-positive size or bad enum)";
    case KDA_ERR_UNSUPPORTED: return "unsupported configuration (head dims, chunk size or sizes)";
    case KDA_ERR_MISALIGNED: return "a tensor pointer is not 16-byte aligned";
    case KDA_ERR_CUDA: return "a CUDA runtime call failed";
    case KDA_ERR_TIMEOUT: return "a kernel's bounded wait gave up (device error word set)";
    case KDA_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

int kda_abi_version(void) { return 103; }

kda_status_t kda_forward_chunked(const void *q, const void *k, const void *v, const void *g,
                                 const void *beta, const float *initial_state, void *out,
                                 float *final_state, int B, int T, int H, int dk, int dv,
                                 int chunk, kda_dtype_t io, kda_stream_t stream)
{
    kda_status_t st = check_dims(B, T, H, dk, dv, io);
    if (st != KDA_OK) return st;
    if (chunk != 64) return KDA_ERR_UNSUPPORTED;
    if (T > 0 && (!q || !k || !v || !g || !beta || !out)) return KDA_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, g, beta, initial_state, out, final_state};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_MISALIGNED;
    cudaStream_t s = (cudaStream_t)stream;
    if (T == 0) return cuda_status(kda::launch_fill_state(initial_state, final_state,
                                                          (size_t)B * H * dk * dv, s));
    kda::ChunkArgs a{q, k, v, g, beta, initial_state, out, final_state, B, T, H, dk, dv,
                     io_of(io), false, false, false, false, error_word()};
    return launch_chunked(a, s);
}

kda_status_t kda_backward_workspace_size(int B, int T, int H, int dk, int dv, kda_dtype_t io,
                                         size_t *bytes)
{
    if (!bytes) return KDA_ERR_INVALID_ARG;
    kda_status_t st = check_dims(B, T, H, dk, dv, io);
    if (st != KDA_OK) return st;
    if (dk != dv) return KDA_ERR_UNSUPPORTED;
    *bytes = kda::backward_workspace_bytes(B, T, H, dk);
    return KDA_OK;
}

kda_status_t kda_backward_chunked(const void *q, const void *k, const void *v, const void *g,
                                  const void *beta, const float *initial_state, const void *d_out,
                                  const float *d_final_state, void *dq, void *dk_, void *dv_, void *dg,
                                  void *dbeta, float *d_initial_state, void *workspace,
                                  size_t workspace_bytes, int B, int T, int H, int dk, int dv,
                                  kda_dtype_t io, kda_stream_t stream)
{
    kda_status_t st = check_dims(B, T, H, dk, dv, io);
    if (st != KDA_OK) return st;
    if (dk != dv) return KDA_ERR_UNSUPPORTED;
    if (T > 0 && (!q || !k || !v || !g || !beta || !d_out || !dq || !dk_ || !dv_ || !dg || !dbeta))
        return KDA_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, g, beta, initial_state, d_out, d_final_state, dq, dk_, dv_, dg, dbeta,
                          d_initial_state};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_MISALIGNED;
    cudaStream_t s = (cudaStream_t)stream;
    if (T == 0) return cuda_status(kda::launch_fill_state(d_final_state, d_initial_state,
                                                          (size_t)B * H * dk * dv, s));
    const size_t need = kda::backward_workspace_bytes(B, T, H, dk);
    if (!workspace || workspace_bytes < need) return KDA_ERR_WORKSPACE;
    if (((uintptr_t)workspace & 255u) != 0) return KDA_ERR_MISALIGNED;
    kda::BackwardArgs a{q, k, v, g, beta, initial_state, d_out, d_final_state, dq, dk_, dv_, dg, dbeta,
                        d_initial_state, (float *)workspace, B, T, H, dk, io_of(io)};
    return cuda_status(kda::launch_backward(a, s));
}

kda_status_t kda_forward_chunked_varlen(const void *q, const void *k, const void *v, const void *g,
                                        const void *beta, const float *initial_state, void *out,
                                        float *final_state, const int *cu_seqlens, int N,
                                        int T_total, int H, int dk, int dv, int chunk,
                                        kda_dtype_t io, kda_stream_t stream)
{
    kda_status_t st = check_dims(N, T_total, H, dk, dv, io);
    if (st != KDA_OK) return st;
    if ((long long)N * H > INT32_MAX / 2) return KDA_ERR_UNSUPPORTED;
    if (chunk != 64) return KDA_ERR_UNSUPPORTED;
    if (!cu_seqlens) return KDA_ERR_INVALID_ARG;
    if (T_total > 0 && (!q || !k || !v || !g || !beta || !out)) return KDA_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, g, beta, initial_state, out, final_state, cu_seqlens};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_MISALIGNED;
    cudaStream_t s = (cudaStream_t)stream;
    if (T_total == 0) return cuda_status(kda::launch_fill_state(initial_state, final_state,
                                                                (size_t)N * H * dk * dv, s));
    // the kernels take B = N sequences over a token axis of T = T_total rows
    kda::ChunkArgs a{q, k, v, g, beta, initial_state, out, final_state, N, T_total, H, dk, dv,
                     io_of(io), false, false, false, false, error_word(), cu_seqlens};
    return launch_chunked(a, s);
}

kda_status_t kda_decode_step(const void *q, const void *k, const void *v, const void *g,
                             const void *beta, float *state, void *out, int B, int H, int dk,
                             int dv, kda_dtype_t io, kda_stream_t stream)
{
    kda_status_t st = check_dims(B, 1, H, dk, dv, io);
    if (st != KDA_OK) return st;
    if (!q || !k || !v || !g || !beta || !state || !out) return KDA_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, g, beta, state, out};
    for (const void *p : ptrs)
        if (!aligned16(p)) return KDA_ERR_MISALIGNED;
    kda::DecodeArgs a{q, k, v, g, beta, state, out, B, H, dk, dv, io_of(io)};
    return cuda_status(kda::launch_decode(a, (cudaStream_t)stream));
}

kda_status_t kda_layer_workspace_size(int B, int T, int H, int dk, int dv, kda_dtype_t io,
                                      size_t *bytes)
{
    if (!bytes) return KDA_ERR_INVALID_ARG;
    kda_status_t st = check_dims(B, T, H, dk, dv, io);
    if (st != KDA_OK) return st;
    *bytes = (T == 0 || layer_on_tensor_cores(io, dk, dv)) ? 0 : layer_workspace(B, T, H, dk, dv).total;
    return KDA_OK;
}

kda_status_t kda_layer_forward(const void *q_raw, const void *k_raw, const void *v_raw,
                               const float *conv_q, const float *conv_k, const float *conv_v,
                               const void *g_raw, const float *A_log, const float *dt_bias,
                               float gate_lower_bound, const void *b_raw, const void *o_gate_raw,
                               const float *o_norm_w, float norm_eps, const float *initial_state,
                               void *out, float *final_state, void *workspace, size_t workspace_bytes,
                               int B, int T, int H, int dk, int dv, kda_dtype_t io,
                               kda_stream_t stream)
{
    kda_status_t st = check_dims(B, T, H, dk, dv, io);
    if (st != KDA_OK) return st;
    return layer_core(q_raw, k_raw, v_raw, conv_q, conv_k, conv_v, g_raw, A_log, dt_bias, gate_lower_bound, b_raw,
                      o_gate_raw, o_norm_w, norm_eps, initial_state, out, final_state, workspace, workspace_bytes, B,
                      T, H, dk, dv, io, stream, nullptr);
}

kda_status_t kda_layer_forward_varlen(const void *q_raw, const void *k_raw, const void *v_raw,
                                      const float *conv_q, const float *conv_k, const float *conv_v,
                                      const void *g_raw, const float *A_log, const float *dt_bias,
                                      float gate_lower_bound, const void *b_raw, const void *o_gate_raw,
                                      const float *o_norm_w, float norm_eps, const float *initial_state,
                                      void *out, float *final_state, const int *cu_seqlens, void *workspace,
                                      size_t workspace_bytes, int N, int T_total, int H, int dk, int dv,
                                      kda_dtype_t io, kda_stream_t stream)
{
    kda_status_t st = check_dims(1, T_total, H, dk, dv, io);
    if (st != KDA_OK) return st;
    if (N < 1) return KDA_ERR_INVALID_ARG;
    if ((long long)N * H > INT32_MAX / 2) return KDA_ERR_UNSUPPORTED;
    if (!cu_seqlens) return KDA_ERR_INVALID_ARG;
    if (!aligned16(cu_seqlens)) return KDA_ERR_MISALIGNED;
    return layer_core(q_raw, k_raw, v_raw, conv_q, conv_k, conv_v, g_raw, A_log, dt_bias, gate_lower_bound, b_raw,
                      o_gate_raw, o_norm_w, norm_eps, initial_state, out, final_state, workspace, workspace_bytes, N,
                      T_total, H, dk, dv, io, stream, cu_seqlens);
}

kda_status_t kda_layer_decode_step(const void *q_raw, const void *k_raw, const void *v_raw,
                                   const float *conv_q, const float *conv_k, const float *conv_v,
                                   void *cache_q, void *cache_k, void *cache_v, const void *g_raw,
                                   const float *A_log, const float *dt_bias, float gate_lower_bound,
                                   const void *b_raw, const void *o_gate_raw, const float *o_norm_w,
                                   float norm_eps, float *state, void *out, int B, int H, int dk, int dv,
                                   kda_dtype_t io, kda_stream_t stream)
{
    kda_status_t st = check_dims(B, 1, H, dk, dv, io);
    if (st != KDA_OK) return st;
    if (dk != 128 || dv != 128) return KDA_ERR_UNSUPPORTED;
    if (!(norm_eps >= 0.0f) || !(gate_lower_bound <= 0.0f)) return KDA_ERR_INVALID_ARG;
    if (!q_raw || !k_raw || !v_raw || !conv_q || !conv_k || !conv_v || !cache_q || !cache_k || !cache_v ||
        !g_raw || !A_log || !b_raw || !o_gate_raw || !state || !out)
        return KDA_ERR_INVALID_ARG;
    const void *ptrs[] = {q_raw, k_raw, v_raw, conv_q, conv_k, conv_v, cache_q, cache_k, cache_v, g_raw,
                          A_log, dt_bias, b_raw, o_gate_raw, o_norm_w, state, out};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_MISALIGNED;
    kda::LayerDecodeArgs a{q_raw, k_raw, v_raw, cache_q, cache_k, cache_v, conv_q, conv_k, conv_v,
                           g_raw, A_log, dt_bias, gate_lower_bound, b_raw, o_gate_raw, o_norm_w,
                           norm_eps, state, out, B, H, io_of(io)};
    return cuda_status(kda::launch_layer_decode(a, (cudaStream_t)stream));
}

kda_status_t kda_set_wait_test_hooks(unsigned long long wait_limit_ns, int skip_load_chunk)
{
    kda::set_wait_hooks(wait_limit_ns, skip_load_chunk);
    return KDA_OK;
}

kda_status_t kda_check_device_error(kda_stream_t stream)
{
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    int *p = error_word();
    if (!p) return KDA_ERR_CUDA;
    int word = 0;
    if (cudaMemcpy(&word, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return KDA_ERR_CUDA;
    if (word != 0) {
        const int zero = 0;
        if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return KDA_ERR_CUDA;
        return KDA_ERR_TIMEOUT;
    }
    return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // extern "C"
