// layer_decode.cu — one decode step of the whole KDA layer core, with a conv-state cache.
//
// Per sequence b and head h, for the new token t (dk = dv = 128):
//   y_X[c] = SiLU(w_X[c,0] x[t-3,c] + w_X[c,1] x[t-2,c] + w_X[c,2] x[t-1,c] + w_X[c,3] x[t,c])
//            for X = q, k, v, with x[t-3..t-1] taken from the conv cache, which then shifts in x[t]
//   q^ = y_q / sqrt(|y_q|^2 + 1e-6),  k^ likewise,  v = y_v
//   g = max(-exp(A_log[h]) softplus(g_raw + dt_bias), lb),  beta = sigmoid(b_raw)
//   S' = Diag(exp g) S;  u = beta (v - S'^T k^);  S <- S' + k^ u^T;  o = S^T q^
//   out = gain * cast_io(o * rsqrt(mean(o^2) + eps)) * sigmoid(o_gate_raw)
// — the same steps as the prefill path (prologue, recurrence, epilogue: the short-conv and
// gate entries of the Kimi-K3 linear-attention config, the KimiRMSNorm excerpt and the
// sigmoid output gate), for the one token a decode step adds.  The fixed-size state and a
// three-token conv history per channel are all a decoding sequence carries.
//
// One CTA of 512 threads per (b, h).  The 64 KB state slice is loaded first (8 float4 per
// thread, 32 threads per 512-byte row), so its latency overlaps the prologue; the column
// sums S'^T k^ and S'^T q^ reduce across the 16 row groups in shared memory; the state is
// written back in place, all in fp32.
#include "common.cuh"
#include "internal.h"

namespace kda {
namespace {

constexpr int LD_THREADS = 512;
constexpr int LD_D = 128;
constexpr int LD_ROWS = LD_THREADS / 32;        // rows per pass: 32 threads per row of 128 floats
constexpr int LD_NPASS = LD_D / LD_ROWS;        // 8
constexpr float LD_L2_EPS = 1e-6f;

template <typename IO>
__global__ void __launch_bounds__(LD_THREADS)
kda_layer_decode_kernel(LayerDecodeArgs a)
{
    __shared__ float s_y[3][LD_D];              // conv + SiLU outputs for q, k, v
    __shared__ float s_alpha[LD_D];
    __shared__ float s_part[3][4];              // per-warp sum q^2, k^2, q.k
    __shared__ __align__(16) float s_red_a[LD_ROWS][LD_D];
    __shared__ __align__(16) float s_red_b[LD_ROWS][LD_D];
    __shared__ float s_u[LD_D];
    __shared__ float s_opart[4];
    __shared__ float s_beta;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x, b = bh / a.H, h = bh % a.H;
    const size_t HD = (size_t)a.H * LD_D;

    // ---------------------------------------------------------------- state loads first
    const int col4 = lane * 4, row0 = warp;
    float *Sb = a.state + (size_t)bh * LD_D * LD_D + col4;
    float4 s[LD_NPASS];
#pragma unroll
    for (int p = 0; p < LD_NPASS; ++p) s[p] = *reinterpret_cast<const float4 *>(Sb + (size_t)(row0 + LD_ROWS * p) * LD_D);

    // ---------------------------------------------------------------- prologue
    if (tid < 3 * LD_D) {
        // tensor X = tid / 128 (q, k, v), channel c = tid % 128
        const int X = tid >> 7, c = tid & (LD_D - 1);
        const IO *xr = X == 0 ? (const IO *)a.q_raw : (X == 1 ? (const IO *)a.k_raw : (const IO *)a.v_raw);
        IO *cache = X == 0 ? (IO *)a.cache_q : (X == 1 ? (IO *)a.cache_k : (IO *)a.cache_v);
        const float *w = X == 0 ? a.conv_q : (X == 1 ? a.conv_k : a.conv_v);
        const size_t ch = (size_t)h * LD_D + c;
        const IO x0 = cache[(size_t)b * 3 * HD + ch], x1 = cache[((size_t)b * 3 + 1) * HD + ch];
        const IO x2 = cache[((size_t)b * 3 + 2) * HD + ch], xt = xr[(size_t)b * HD + ch];
        const float4 wv = *reinterpret_cast<const float4 *>(w + ch * 4);
        float acc = wv.x * to_f32(x0);
        acc += wv.y * to_f32(x1);
        acc += wv.z * to_f32(x2);
        acc += wv.w * to_f32(xt);
        const float y = siluf_(acc);
        s_y[X][c] = y;
        // the cache shifts in the new raw token (exact copies in the I/O dtype)
        cache[(size_t)b * 3 * HD + ch] = x1;
        cache[((size_t)b * 3 + 1) * HD + ch] = x2;
        cache[((size_t)b * 3 + 2) * HD + ch] = xt;
        if (X < 2) {
            const float ss = warp_sum(y * y);
            if (lane == 0) s_part[X][warp & 3] = ss;
        }
    } else if (tid < 3 * LD_D + LD_D) {
        // gate g = max(-exp(A_log[h]) softplus(g_raw + dt_bias), lb) for channel c; alpha = exp(g)
        const int c = tid - 3 * LD_D;
        const float bias = a.dt_bias ? a.dt_bias[(size_t)h * LD_D + c] : 0.0f;
        const float x = to_f32(((const IO *)a.g_raw)[(size_t)bh * LD_D + c]);
        s_alpha[c] = __expf(fmaxf(-__expf(a.A_log[h]) * softplusf_(x + bias), a.g_lb));
        if (c == 0) s_beta = sigmoidf_(to_f32(((const IO *)a.b_raw)[bh]));
    }
    __syncthreads();
    if (warp < 4) {
        const float qk = warp_sum(s_y[0][tid] * s_y[1][tid]);
        if (lane == 0) s_part[2][warp] = qk;
    }
    __syncthreads();
    const float rq = rsqrtf(s_part[0][0] + s_part[0][1] + s_part[0][2] + s_part[0][3] + LD_L2_EPS);
    const float rk = rsqrtf(s_part[1][0] + s_part[1][1] + s_part[1][2] + s_part[1][3] + LD_L2_EPS);

    // ---------------------------------------------------------------- decay, column sums
    float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int p = 0; p < LD_NPASS; ++p) {
        const int r = row0 + LD_ROWS * p;
        const float al = s_alpha[r], kr = s_y[1][r] * rk, qr = s_y[0][r] * rq;
        s[p].x *= al; s[p].y *= al; s[p].z *= al; s[p].w *= al;
        sa[0] += kr * s[p].x; sa[1] += kr * s[p].y; sa[2] += kr * s[p].z; sa[3] += kr * s[p].w;
        sb[0] += qr * s[p].x; sb[1] += qr * s[p].y; sb[2] += qr * s[p].z; sb[3] += qr * s[p].w;
    }
    *reinterpret_cast<float4 *>(&s_red_a[row0][col4]) = make_float4(sa[0], sa[1], sa[2], sa[3]);
    *reinterpret_cast<float4 *>(&s_red_b[row0][col4]) = make_float4(sb[0], sb[1], sb[2], sb[3]);
    __syncthreads();

    // ---------------------------------------------------------------- u, o and the epilogue
    float o = 0.0f;
    if (tid < LD_D) {
        float ka = 0.f, qb = 0.f;
#pragma unroll
        for (int w = 0; w < LD_ROWS; ++w) {
            ka += s_red_a[w][tid];
            qb += s_red_b[w][tid];
        }
        const float qk = (s_part[2][0] + s_part[2][1] + s_part[2][2] + s_part[2][3]) * rq * rk;
        const float u = s_beta * (s_y[2][tid] - ka);
        s_u[tid] = u;
        o = qb + qk * u;   // S_new^T q^ = S'^T q^ + (q^ . k^) u
        const float ss = warp_sum(o * o);
        if (lane == 0) s_opart[warp] = ss;
    }
    __syncthreads();
    if (tid < LD_D) {
        const float r = rsqrtf((s_opart[0] + s_opart[1] + s_opart[2] + s_opart[3]) / (float)LD_D + a.eps);
        float y = to_f32(from_f32<IO>(o * r));   // cast to the activation dtype, then gain
        if (a.gain) y *= a.gain[tid];
        const float z = to_f32(((const IO *)a.o_gate_raw)[(size_t)bh * LD_D + tid]);
        ((IO *)a.out)[(size_t)bh * LD_D + tid] = from_f32<IO>(y * sigmoidf_(z));
    }

    // ---------------------------------------------------------------- S <- S' + k^ u^T
    const float u0 = s_u[col4], u1 = s_u[col4 + 1], u2 = s_u[col4 + 2], u3 = s_u[col4 + 3];
#pragma unroll
    for (int p = 0; p < LD_NPASS; ++p) {
        const int r = row0 + LD_ROWS * p;
        const float kr = s_y[1][r] * rk;
        *reinterpret_cast<float4 *>(Sb + (size_t)r * LD_D) =
            make_float4(s[p].x + kr * u0, s[p].y + kr * u1, s[p].z + kr * u2, s[p].w + kr * u3);
    }
}

}  // namespace

cudaError_t launch_layer_decode(const LayerDecodeArgs &a, cudaStream_t s)
{
    if (a.io == IO_F32) kda_layer_decode_kernel<float><<<a.B * a.H, LD_THREADS, 0, s>>>(a);
    else kda_layer_decode_kernel<__nv_bfloat16><<<a.B * a.H, LD_THREADS, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace kda
