// internal.h — host-side launcher interface between the C ABI (api.cu) and the kernels.
// Launchers assume validated arguments; they only configure and launch.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>

#include <mutex>

namespace kda {

enum IoType { IO_F32 = 0, IO_BF16 = 1 };

// Chunked prefill operands.  q, k, g, v, beta, out are in `io` dtype unless the
// *_f32 flags say the operand is float32 (used by the layer path for its
// internally computed gate and beta).
struct ChunkArgs {
    const void *q, *k, *v, *g, *beta;
    const float *s0;  // nullable
    void *out;
    float *sT;        // nullable
    int B, T, H, dk, dv;
    IoType io;
    bool qkv_f32, g_f32, beta_f32, out_f32;
    int *err;
    const int *cu = nullptr;  // packed variable length: sequence offsets [B + 1], device; T = total tokens
};

struct DecodeArgs {
    const void *q, *k, *v, *g, *beta;
    float *state;
    void *out;
    int B, H, dk, dv;
    IoType io;
};

struct PrologueArgs {
    const void *q_raw, *k_raw, *v_raw, *g_raw, *b_raw;
    const float *conv_q, *conv_k, *conv_v, *A_log, *dt_bias;
    float g_lb;                   // lower bound on the log-decay g (-inf: none)
    float *q, *k, *v, *g, *beta;  // workspace outputs, fp32
    int B, T, H, dk, dv;
    IoType io;
    const int *cu = nullptr;      // packed sequences: offsets [nseq + 1], device (B = 1, T = total)
    int nseq = 0;
};

struct EpilogueArgs {
    const float *o;  // [B, T, H, dv] fp32
    const void *z;   // o_gate_raw, io dtype
    const float *gain;
    float eps;
    void *out;
    int B, T, H, dv;
    IoType io;
};

// One decode step of the whole layer core (conv cache + prologue + recurrence + epilogue).
struct LayerDecodeArgs {
    const void *q_raw, *k_raw, *v_raw;      // [B, H*128], io
    void *cache_q, *cache_k, *cache_v;      // [B, 3, H*128], io, in place (oldest tap first)
    const float *conv_q, *conv_k, *conv_v;  // [H*128, 4]
    const void *g_raw;                      // [B, H, 128], io
    const float *A_log, *dt_bias;           // [H]; [H*128] or null
    float g_lb;                             // lower bound on the log-decay g (-inf: none)
    const void *b_raw, *o_gate_raw;         // [B, H]; [B, H, 128], io
    const float *gain;                      // [128] or null
    float eps;
    float *state;                           // [B, H, 128, 128] fp32, in place
    void *out;                              // [B, H, 128], io
    int B, H;
    IoType io;
};
cudaError_t launch_layer_decode(const LayerDecodeArgs &a, cudaStream_t s);

// The whole layer core (prologue, chunked recurrence, epilogue) in one tcgen05 kernel: bf16
// I/O, dk = dv = 128, no workspace.
struct LayerTcArgs {
    const void *q_raw, *k_raw, *v_raw, *g_raw, *b_raw, *o_gate_raw;   // bf16 [B, T, H, 128] / [B, T, H]
    const float *conv_q, *conv_k, *conv_v, *A_log, *dt_bias, *gain;
    float g_lb, eps;
    const float *s0;
    float *sT;
    void *out;
    int B, T, H, dk, dv;   // packed: B = sequences over a token axis of T rows
    IoType io;
    int *err;
    const int *cu;
};
bool layer_tc_supported(const LayerTcArgs &a);
cudaError_t launch_layer_tc(const LayerTcArgs &a, cudaStream_t s);

// CUDA-core chunked kernel: any supported dtype, dk, dv in {64, 128}.
cudaError_t launch_chunk_simt(const ChunkArgs &a, cudaStream_t s);
// Exact fp32 chunked kernel on CUDA cores for dk = dv = 128 with all-fp32 operands.
cudaError_t launch_chunk_f32(const ChunkArgs &a, cudaStream_t s);
bool chunk_f32_supported(const ChunkArgs &a);
// tcgen05 chunked kernel: bf16 I/O, dk = dv = 128.
cudaError_t launch_chunk_tc(const ChunkArgs &a, cudaStream_t s);
bool chunk_tc_supported(const ChunkArgs &a);

// [B, T, H, 128] bf16 -> 4-D TMA map (128, H, T, B) with box (64, 1, box_rows, 1), 128-byte
// swizzle and zero fill past the extents.  False if the driver entry point is missing.
bool make_tile_map(CUtensorMap *m, const void *base, int B, int T, int H, int box_rows);
// The current device is sm_100 (B200); the driver provides cuTensorMapEncodeTiled.
bool device_is_sm100();
bool tensor_maps_available();

// Limit of every bounded mbarrier wait in the tensor-core kernels, and an injected failure
// (the tile load of chunk `skip_load_chunk` is never issued; -1: none).  Process-wide, read at
// each launch; set through kda_set_wait_test_hooks.
struct WaitHooks {
    unsigned long long wait_ns;
    int skip_load_chunk;
};
constexpr unsigned long long kDefaultWaitNs = 2000000000ull;
WaitHooks wait_hooks();
void set_wait_hooks(unsigned long long wait_ns, int skip_load_chunk);

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s);
cudaError_t launch_prologue(const PrologueArgs &a, cudaStream_t s);
cudaError_t launch_epilogue(const EpilogueArgs &a, cudaStream_t s);
cudaError_t launch_fill_state(const float *s0, float *sT, size_t n, cudaStream_t s);

// Opts `fn` into `bytes` of dynamic shared memory on the current device.  The attribute
// belongs to the device's context, so it is set once per device (a process may drive
// several GPUs); Tag makes the flags distinct per kernel.
constexpr int kMaxSmemDevices = 64;
template <typename Tag>
cudaError_t smem_opt_in(const void *fn, int bytes)
{
    static std::once_flag once[kMaxSmemDevices];
    static cudaError_t err[kMaxSmemDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    if (dev < 0 || dev >= kMaxSmemDevices) return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    std::call_once(once[dev], [&] { err[dev] = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes); });
    return err[dev];
}

// Gradients of the recurrence (dk = dv = d).
struct BackwardArgs {
    const void *q, *k, *v, *g, *beta;   // io dtype, [B, T, H, d] / [B, T, H]
    const float *s0;                    // nullable
    const void *dO;                     // io dtype
    const float *dST;                   // nullable
    void *dq, *dk, *dv, *dg, *dbeta;    // io dtype
    float *ds0;                         // nullable
    float *ckpt;                        // backward_workspace_bytes()
    int B, T, H, d;
    IoType io;
};
size_t backward_workspace_bytes(int B, int T, int H, int d);
cudaError_t launch_backward(const BackwardArgs &a, cudaStream_t s);

}  // namespace kda
