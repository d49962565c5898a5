// layer_simt.cu — KDA layer prologue and epilogue as streaming CUDA-core kernels.
//
// Prologue, per (b, t, h) token-head (one warp each):
//   q = l2norm(SiLU(conv_q * q_raw)),  k = l2norm(SiLU(conv_k * k_raw)),  v = SiLU(conv_v * v_raw)
//     depthwise causal conv of kernel 4 with zero history, PyTorch Conv1d tap order:
//     y[t, c] = sum_{i=0..3} w[c, i] x[t - 3 + i, c]
//     (open-model-atlas "Kimi-K3" linear_attn_config: short_conv_kernel_size 4;
//      maxtext PR #5548 review item 2: {q,k,v}_conv1d.weight [heads*d, 1, 4] in F32)
//   g = -exp(A_log[h]) softplus(g_raw + dt_bias[h, c]),  beta = sigmoid(b_raw)
//     (maxtext PR #5548 review item 2: exp(A_log) drives the state decay)
// Epilogue, per (b, t, h) row of dv values (one warp each):
//   out = gain * cast_io(o * rsqrt(mean(o^2) + eps)) * sigmoid(z)
//     (atlas.klimoza.dev KimiRMSNorm excerpt; maxtext PR #5543 sigmoid output gate)
// Intermediates are fp32 so the log-decay keeps full precision before its
// cumulative sums.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace kda {
namespace {

constexpr int LY_THREADS = 256;
constexpr float L2_EPS = 1e-6f;

template <typename IO, int D>
KDA_DEVICE void conv_row(const IO *__restrict__ x, const float *__restrict__ w, int t, size_t row_stride,
                         int c0, float (&y)[D / 32])
{
    // x points at (b, t=0, channel h*D); lane handles channels c0 + 32*e
#pragma unroll
    for (int e = 0; e < D / 32; ++e) {
        const int c = c0 + 32 * e;
        const float4 wc = *reinterpret_cast<const float4 *>(w + (size_t)c * 4);
        float acc = 0.0f;
        if (t >= 3) acc += wc.x * to_f32(x[(size_t)(t - 3) * row_stride + c]);
        if (t >= 2) acc += wc.y * to_f32(x[(size_t)(t - 2) * row_stride + c]);
        if (t >= 1) acc += wc.z * to_f32(x[(size_t)(t - 1) * row_stride + c]);
        acc += wc.w * to_f32(x[(size_t)t * row_stride + c]);
        y[e] = siluf_(acc);
    }
}

template <typename IO, int DK, int DV>
__global__ void __launch_bounds__(LY_THREADS)
kda_prologue_kernel(PrologueArgs a)
{
    const int warp = (blockIdx.x * LY_THREADS + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const long long ntok = (long long)a.B * a.T * a.H;
    if (warp >= ntok) return;
    const int h = warp % a.H;
    const long long bt = warp / a.H;
    const int t = (int)(bt % a.T);
    const long long b = bt / a.T;
    const size_t rsk = (size_t)a.H * DK, rsv = (size_t)a.H * DV;

    // q, k: conv + SiLU + L2-norm over the head's dk channels
    {
        const IO *xq = (const IO *)a.q_raw + (size_t)b * a.T * rsk + (size_t)h * DK;
        const IO *xk = (const IO *)a.k_raw + (size_t)b * a.T * rsk + (size_t)h * DK;
        float yq[DK / 32], yk[DK / 32];
        conv_row<IO, DK>(xq, a.conv_q + (size_t)h * DK * 4, t, rsk, lane, yq);
        conv_row<IO, DK>(xk, a.conv_k + (size_t)h * DK * 4, t, rsk, lane, yk);
        float sq = 0.f, sk = 0.f;
#pragma unroll
        for (int e = 0; e < DK / 32; ++e) { sq += yq[e] * yq[e]; sk += yk[e] * yk[e]; }
        sq = rsqrtf(warp_sum(sq) + L2_EPS);
        sk = rsqrtf(warp_sum(sk) + L2_EPS);
        const size_t o = (size_t)warp * DK;
#pragma unroll
        for (int e = 0; e < DK / 32; ++e) {
            a.q[o + lane + 32 * e] = yq[e] * sq;
            a.k[o + lane + 32 * e] = yk[e] * sk;
        }
    }
    // v: conv + SiLU
    {
        const IO *xv = (const IO *)a.v_raw + (size_t)b * a.T * rsv + (size_t)h * DV;
        float yv[DV / 32];
        conv_row<IO, DV>(xv, a.conv_v + (size_t)h * DV * 4, t, rsv, lane, yv);
        const size_t o = (size_t)warp * DV;
#pragma unroll
        for (int e = 0; e < DV / 32; ++e) a.v[o + lane + 32 * e] = yv[e];
    }
    // gate and beta
    {
        const float scale = __expf(a.A_log[h]);
        const IO *gr = (const IO *)a.g_raw + (size_t)warp * DK;
#pragma unroll
        for (int e = 0; e < DK / 32; ++e) {
            const int c = lane + 32 * e;
            const float bias = a.dt_bias ? a.dt_bias[(size_t)h * DK + c] : 0.0f;
            a.g[(size_t)warp * DK + c] = -scale * softplusf_(to_f32(gr[c]) + bias);
        }
        if (lane == 0) a.beta[warp] = sigmoidf_(to_f32(((const IO *)a.b_raw)[warp]));
    }
}

template <typename IO, int DV>
__global__ void __launch_bounds__(LY_THREADS)
kda_epilogue_kernel(EpilogueArgs a)
{
    const int warp = (blockIdx.x * LY_THREADS + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const long long nrow = (long long)a.B * a.T * a.H;
    if (warp >= nrow) return;
    const float *o = a.o + (size_t)warp * DV;
    float x[DV / 32];
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < DV / 32; ++e) { x[e] = o[lane + 32 * e]; ss += x[e] * x[e]; }
    const float r = rsqrtf(warp_sum(ss) / (float)DV + a.eps);
    const IO *z = (const IO *)a.z + (size_t)warp * DV;
    IO *out = (IO *)a.out + (size_t)warp * DV;
#pragma unroll
    for (int e = 0; e < DV / 32; ++e) {
        const int c = lane + 32 * e;
        float y = to_f32(from_f32<IO>(x[e] * r));   // cast back to the activation dtype
        if (a.gain) y *= a.gain[c];
        out[c] = from_f32<IO>(y * sigmoidf_(to_f32(z[c])));
    }
}

__global__ void kda_fill_state_kernel(const float *__restrict__ s0, float *__restrict__ sT, size_t n)
{
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
        sT[i] = s0 ? s0[i] : 0.0f;
}

template <typename IO, int DK>
cudaError_t launch_pro_dk(const PrologueArgs &a, cudaStream_t s)
{
    const long long warps = (long long)a.B * a.T * a.H;
    const unsigned blocks = (unsigned)((warps * 32 + LY_THREADS - 1) / LY_THREADS);
    if (a.dv == 64) kda_prologue_kernel<IO, DK, 64><<<blocks, LY_THREADS, 0, s>>>(a);
    else kda_prologue_kernel<IO, DK, 128><<<blocks, LY_THREADS, 0, s>>>(a);
    return cudaGetLastError();
}

template <typename IO>
cudaError_t launch_epi_t(const EpilogueArgs &a, cudaStream_t s)
{
    const long long warps = (long long)a.B * a.T * a.H;
    const unsigned blocks = (unsigned)((warps * 32 + LY_THREADS - 1) / LY_THREADS);
    if (a.dv == 64) kda_epilogue_kernel<IO, 64><<<blocks, LY_THREADS, 0, s>>>(a);
    else kda_epilogue_kernel<IO, 128><<<blocks, LY_THREADS, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prologue(const PrologueArgs &a, cudaStream_t s)
{
    using bf = __nv_bfloat16;
    if (a.io == IO_F32) return a.dk == 64 ? launch_pro_dk<float, 64>(a, s) : launch_pro_dk<float, 128>(a, s);
    return a.dk == 64 ? launch_pro_dk<bf, 64>(a, s) : launch_pro_dk<bf, 128>(a, s);
}

cudaError_t launch_epilogue(const EpilogueArgs &a, cudaStream_t s)
{
    return a.io == IO_F32 ? launch_epi_t<float>(a, s) : launch_epi_t<__nv_bfloat16>(a, s);
}

cudaError_t launch_fill_state(const float *s0, float *sT, size_t n, cudaStream_t s)
{
    if (n == 0 || sT == nullptr || s0 == sT) return cudaSuccess;
    const unsigned blocks = (unsigned)std::min<size_t>((n + 255) / 256, 148 * 16);
    kda_fill_state_kernel<<<blocks, 256, 0, s>>>(s0, sT, n);
    return cudaGetLastError();
}

}  // namespace kda
