// layer_simt.cu — KDA layer prologue and epilogue as streaming CUDA-core kernels.
//
// Prologue, per (b, h) and run of 8 tokens (one warp each):
//   q = l2norm(SiLU(conv_q * q_raw)),  k = l2norm(SiLU(conv_k * k_raw)),  v = SiLU(conv_v * v_raw)
//     depthwise causal conv of kernel 4 with zero history, PyTorch Conv1d tap order:
//     y[t, c] = sum_{i=0..3} w[c, i] x[t - 3 + i, c]
//     (open-model-atlas "Kimi-K3" linear_attn_config: short_conv_kernel_size 4;
//      maxtext PR #5548 review item 2: {q,k,v}_conv1d.weight [heads*d, 1, 4] in F32)
//   g = max(-exp(A_log[h]) softplus(g_raw + dt_bias[h, c]), lb),  beta = sigmoid(b_raw)
//     (lb: the linear-attention config's gate_lower_bound, read as a bound on g itself)
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

constexpr int RUN = 8;   // tokens per warp in the prologue

// N consecutive elements (N = 2 or 4) as floats, and N floats stored
template <int N> KDA_DEVICE void ldn(const float *p, float (&o)[N])
{
    if constexpr (N == 4) {
        const float4 t = *reinterpret_cast<const float4 *>(p);
        o[0] = t.x; o[1] = t.y; o[2] = t.z; o[3] = t.w;
    } else {
        const float2 t = *reinterpret_cast<const float2 *>(p);
        o[0] = t.x; o[1] = t.y;
    }
}
template <int N> KDA_DEVICE void ldn(const __nv_bfloat16 *p, float (&o)[N])
{
    if constexpr (N == 4) {
        ld4(p, o);
    } else {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p));
        o[0] = f.x; o[1] = f.y;
    }
}
template <int N> KDA_DEVICE void stn(float *p, const float (&v)[N])
{
    if constexpr (N == 4) *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    else *reinterpret_cast<float2 *>(p) = make_float2(v[0], v[1]);
}

// Where the run starting at token t0 sits among packed sequences: lo = first token of its
// sequence (the conv's history floor), nb = first token of the next sequence, si = its index.
// Fixed length: lo = 0, nb = no boundary.  Offsets are clamped into the array, so malformed
// ones cannot send a read out of bounds.
struct SeqPos {
    int lo, nb, si;
};
KDA_DEVICE SeqPos seq_pos(const int *cu, int nseq, int t0)
{
    if (!cu) return SeqPos{0, 0x7fffffff, 0};
    int a = 0, b = nseq - 1;   // the last sequence whose start is <= t0
    while (a < b) {
        const int m = (a + b + 1) >> 1;
        if (cu[m] <= t0) a = m;
        else b = m - 1;
    }
    return SeqPos{cu[a], cu[a + 1], a};
}

// One head's channels of one input stream over a run of tokens t0 .. t0 + nt - 1: causal
// depthwise conv (PyTorch Conv1d tap order: y[t, c] = sum_i w[c, i] x[t - 3 + i, c], zero
// history before each sequence's first token) + SiLU [+ L2-norm over the head's D channels].
// Lane l owns channels N l .. N l + N - 1 and slides a three-row window, so every input row is
// read once; the window restarts from zeros where a packed sequence begins.
template <typename IO, int D, bool NORM>
KDA_DEVICE void conv_stream(const IO *__restrict__ x, size_t rs, const float *__restrict__ w, float *__restrict__ dst,
                            size_t drs, int t0, int nt, int lane, SeqPos sp, const int *cu, int nseq)
{
    constexpr int N = D / 32;
    const int c0 = N * lane;
    float wt[N][4], x3[N], x2[N], x1[N];
#pragma unroll
    for (int e = 0; e < N; ++e) {
        const float4 wv = *reinterpret_cast<const float4 *>(w + (size_t)(c0 + e) * 4);
        wt[e][0] = wv.x; wt[e][1] = wv.y; wt[e][2] = wv.z; wt[e][3] = wv.w;
        x3[e] = x2[e] = x1[e] = 0.0f;
    }
    if (t0 - 3 >= sp.lo) ldn<N>(x + (size_t)(t0 - 3) * rs + c0, x3);
    if (t0 - 2 >= sp.lo) ldn<N>(x + (size_t)(t0 - 2) * rs + c0, x2);
    if (t0 - 1 >= sp.lo) ldn<N>(x + (size_t)(t0 - 1) * rs + c0, x1);
    for (int r = 0; r < nt; ++r) {
        const int t = t0 + r;
        while (t >= sp.nb) {   // a packed sequence starts here (empty ones are stepped over)
#pragma unroll
            for (int e = 0; e < N; ++e) x3[e] = x2[e] = x1[e] = 0.0f;
            ++sp.si;
            sp.nb = sp.si < nseq ? cu[sp.si + 1] : 0x7fffffff;
        }
        float xt[N], y[N];
        ldn<N>(x + (size_t)t * rs + c0, xt);
        float ss = 0.0f;
#pragma unroll
        for (int e = 0; e < N; ++e) {
            float acc = wt[e][0] * x3[e];
            acc += wt[e][1] * x2[e];
            acc += wt[e][2] * x1[e];
            acc += wt[e][3] * xt[e];
            y[e] = siluf_(acc);
            ss += y[e] * y[e];
            x3[e] = x2[e]; x2[e] = x1[e]; x1[e] = xt[e];
        }
        if (NORM) {
            const float sc = rsqrtf(warp_sum(ss) + L2_EPS);
#pragma unroll
            for (int e = 0; e < N; ++e) y[e] *= sc;
        }
        stn<N>(dst + (size_t)t * drs + c0, y);
    }
}

template <typename IO, int DK, int DV>
__global__ void __launch_bounds__(LY_THREADS)
kda_prologue_kernel(PrologueArgs a)
{
    // one warp per (b, h, run of RUN tokens); consecutive warps take consecutive heads
    const long long warp = ((long long)blockIdx.x * LY_THREADS + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int nrun = (a.T + RUN - 1) / RUN;
    if (warp >= (long long)a.B * a.H * nrun) return;
    const int h = (int)(warp % a.H);
    const long long br = warp / a.H;
    const int t0 = (int)(br % nrun) * RUN;
    const int b = (int)(br / nrun);
    const int nt = min(RUN, a.T - t0);
    const size_t rsk = (size_t)a.H * DK, rsv = (size_t)a.H * DV;
    const size_t bt0 = (size_t)b * a.T;   // first (b, t) row of this sequence
    const SeqPos sp = seq_pos(a.cu, a.nseq, t0);

    conv_stream<IO, DK, true>((const IO *)a.q_raw + bt0 * rsk + (size_t)h * DK, rsk, a.conv_q + (size_t)h * DK * 4,
                              a.q + (bt0 * a.H + h) * DK, rsk, t0, nt, lane, sp, a.cu, a.nseq);
    conv_stream<IO, DK, true>((const IO *)a.k_raw + bt0 * rsk + (size_t)h * DK, rsk, a.conv_k + (size_t)h * DK * 4,
                              a.k + (bt0 * a.H + h) * DK, rsk, t0, nt, lane, sp, a.cu, a.nseq);
    conv_stream<IO, DV, false>((const IO *)a.v_raw + bt0 * rsv + (size_t)h * DV, rsv, a.conv_v + (size_t)h * DV * 4,
                               a.v + (bt0 * a.H + h) * DV, rsv, t0, nt, lane, sp, a.cu, a.nseq);
    // gate g = max(-exp(A_log[h]) softplus(g_raw + dt_bias[h, c]), lb) and beta = sigmoid(b_raw)
    {
        constexpr int N = DK / 32;
        const int c0 = N * lane;
        const float scale = __expf(a.A_log[h]);
        float bias[N];
#pragma unroll
        for (int e = 0; e < N; ++e) bias[e] = a.dt_bias ? a.dt_bias[(size_t)h * DK + c0 + e] : 0.0f;
        for (int r = 0; r < nt; ++r) {
            const size_t row = ((bt0 + t0 + r) * a.H + h) * DK + c0;
            float x[N];
            ldn<N>((const IO *)a.g_raw + row, x);
#pragma unroll
            for (int e = 0; e < N; ++e) x[e] = fmaxf(-scale * softplusf_(x[e] + bias[e]), a.g_lb);
            stn<N>(a.g + row, x);
        }
        if (lane < nt) {
            const size_t th = (bt0 + t0 + lane) * a.H + h;
            a.beta[th] = sigmoidf_(to_f32(((const IO *)a.b_raw)[th]));
        }
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
    const long long warps = (long long)a.B * a.H * ((a.T + RUN - 1) / RUN);
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
