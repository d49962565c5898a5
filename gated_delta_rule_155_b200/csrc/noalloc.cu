// noalloc.cu — kda_layer_forward_noalloc: the layer forward with its scratch in a
// fixed, library-owned device buffer instead of a caller-provided workspace.
//
// Who needs it: callers that must not allocate device memory on their call path —
// a serving loop whose device memory is planned once at start-up, a plugin or
// callback interface that hands the code no allocator, or latency-critical code that
// cannot pay for cudaMalloc, which can synchronise the whole device.  Such callers
// still own the inputs and outputs; only the intermediate buffers move here.
//
// The scratch is one file-scope __device__ array of KDA_NOALLOC_SCRATCH_BYTES.  Every
// GPU that loads this library holds it until the process exits.  All calls share it
// and it keeps the last call's contents; the layer pipeline writes every scratch
// byte it reads within the same call, so nothing has to start at zero.  Calls whose
// work overlaps on the GPU (other streams, other host threads) race on the scratch.
//
// In host code the array's name is only a host-side stand-in, not a device address,
// so its device address is looked up once per device with that device current
// (cudaGetSymbolAddress) on the first call made on that device; make that first call
// before any stream capture begins.
#include <mutex>

#include "../../include/kda.h"

namespace {

__device__ __align__(256) unsigned char g_layer_scratch[KDA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::once_flag g_once[kMaxDevices];
void *g_scratch[kMaxDevices];
cudaError_t g_scratch_err[kMaxDevices];

// Device address of the scratch array on the current device, or nullptr.
void *scratch_on_current_device()
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::call_once(g_once[dev], [dev] {
        void *p = nullptr;
        g_scratch_err[dev] = cudaGetSymbolAddress(&p, g_layer_scratch);
        if (g_scratch_err[dev] == cudaSuccess) g_scratch[dev] = p;
        else cudaGetLastError();
    });
    return g_scratch_err[dev] == cudaSuccess ? g_scratch[dev] : nullptr;
}

}  // namespace

extern "C" kda_status_t kda_layer_forward_noalloc(
    const void *q_raw, const void *k_raw, const void *v_raw, const float *conv_q, const float *conv_k,
    const float *conv_v, const void *g_raw, const float *A_log, const float *dt_bias, float gate_lower_bound,
    const void *b_raw,
    const void *o_gate_raw, const float *o_norm_w, float norm_eps, const float *initial_state, void *out,
    float *final_state, int B, int T, int H, int dk, int dv, kda_dtype_t io, kda_stream_t stream)
{
    size_t need = 0;
    kda_status_t st = kda_layer_workspace_size(B, T, H, dk, dv, io, &need);
    if (st != KDA_OK) return st;
    if (need > KDA_NOALLOC_SCRATCH_BYTES) return KDA_ERR_WORKSPACE;  // beyond the built-in maximum
    void *scratch = nullptr;
    if (need > 0) {
        scratch = scratch_on_current_device();
        if (!scratch) return KDA_ERR_CUDA;
    }
    return kda_layer_forward(q_raw, k_raw, v_raw, conv_q, conv_k, conv_v, g_raw, A_log, dt_bias,
                             gate_lower_bound, b_raw,
                             o_gate_raw, o_norm_w, norm_eps, initial_state, out, final_state, scratch,
                             need > 0 ? KDA_NOALLOC_SCRATCH_BYTES : 0, B, T, H, dk, dv, io, stream);
}
