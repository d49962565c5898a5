// decode.cu — single-token KDA decode step (memory-bound, one pass over the fp32 state).
//
// Per (sequence b, head h), with S the dk x dv fp32 state:
//     S' = Diag(exp g) S;   a = S'^T k;   b = S'^T q;   u = beta (v - a)
//     S  <- S' + k u^T;     o = S^T q = b + (q . k) u
// (the gated delta rule for one token; the fixed-size per-head state is what the
//  open-model-atlas "Kimi-K3 ?inspect=blocks" page contrasts with the KV cache).
//
// The state is read once and written once.  At dk = dv = 128 one CTA of 512 threads owns a
// head: a warp reads whole 512-byte rows (one float4 per lane), 16 rows per pass, 8 passes,
// issued before anything else, so 64 KB per CTA are in flight at once; the column sums over dk
// reduce across the 16 row groups in shared memory.  Other shapes: a CTA owns one 64-column
// slice of one head, 256 threads, 16 threads per 256-byte row segment, 16 rows per pass; column
// sums reduce across the two rows a warp holds (shuffle) and then across the 8 warps (smem).
// Either way each thread keeps its decayed float4s in registers between the reduction and the
// write-back.
#include "common.cuh"
#include "internal.h"

namespace kda {
namespace {

constexpr int DEC_THREADS = 256;
constexpr int DEC_SLICE = 64;  // value columns per CTA

template <typename IO, int DK>
__global__ void __launch_bounds__(DEC_THREADS, 3)
kda_decode_kernel(const IO *__restrict__ q, const IO *__restrict__ k, const IO *__restrict__ v,
                  const IO *__restrict__ g, const IO *__restrict__ beta, float *state,
                  IO *__restrict__ out, int H, int dv)
{
    constexpr int ROWS_PER_PASS = DEC_THREADS / 16;  // 16
    constexpr int NPASS = DK / ROWS_PER_PASS;
    __shared__ float s_alpha[DK], s_k[DK], s_q[DK];
    __shared__ float s_red_a[DEC_THREADS / 32][DEC_SLICE];
    __shared__ float s_red_b[DEC_THREADS / 32][DEC_SLICE];
    __shared__ float s_u[DEC_SLICE];
    __shared__ float s_qk;

    const int bh = blockIdx.x;            // b * H + h
    const int v0 = blockIdx.y * DEC_SLICE;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const size_t kvec = (size_t)bh * DK;
    const size_t vvec = (size_t)bh * dv;

    // the state loads go out first, so their latency overlaps the small vector loads below
    const int col = (tid & 15) * 4;       // column offset inside the slice
    const int row0 = tid >> 4;            // 0..15
    float *Sbase = state + (size_t)bh * DK * dv + v0 + col;
    float4 s[NPASS];
#pragma unroll
    for (int p = 0; p < NPASS; ++p) {
        const int r = row0 + p * ROWS_PER_PASS;
        s[p] = *reinterpret_cast<const float4 *>(Sbase + (size_t)r * dv);
    }

    if (tid < DK) {
        s_alpha[tid] = __expf(to_f32(g[kvec + tid]));
        s_k[tid] = to_f32(k[kvec + tid]);
        s_q[tid] = to_f32(q[kvec + tid]);
    }
    __syncthreads();
    if (warp == 0) {
        float p = 0.0f;
        for (int c = lane; c < DK; c += 32) p += s_q[c] * s_k[c];
        p = warp_sum(p);
        if (lane == 0) s_qk = p;
    }

    float a[4] = {0.f, 0.f, 0.f, 0.f}, b[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int p = 0; p < NPASS; ++p) {
        const int r = row0 + p * ROWS_PER_PASS;
        const float al = s_alpha[r], kr = s_k[r], qr = s_q[r];
        s[p].x *= al; s[p].y *= al; s[p].z *= al; s[p].w *= al;
        a[0] += kr * s[p].x; a[1] += kr * s[p].y; a[2] += kr * s[p].z; a[3] += kr * s[p].w;
        b[0] += qr * s[p].x; b[1] += qr * s[p].y; b[2] += qr * s[p].z; b[3] += qr * s[p].w;
    }
    // lanes l and l ^ 16 hold the same columns (rows row0 and row0 + 1)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        a[j] += __shfl_xor_sync(0xffffffffu, a[j], 16);
        b[j] += __shfl_xor_sync(0xffffffffu, b[j], 16);
    }
    if (lane < 16) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            s_red_a[warp][col + j] = a[j];
            s_red_b[warp][col + j] = b[j];
        }
    }
    __syncthreads();
    if (tid < DEC_SLICE) {
        float sa = 0.f, sb = 0.f;
#pragma unroll
        for (int w = 0; w < DEC_THREADS / 32; ++w) {
            sa += s_red_a[w][tid];
            sb += s_red_b[w][tid];
        }
        const float bt = to_f32(beta[bh]);
        const float u = bt * (to_f32(v[vvec + v0 + tid]) - sa);
        s_u[tid] = u;
        out[vvec + v0 + tid] = from_f32<IO>(sb + s_qk * u);
    }
    __syncthreads();
    const float u0 = s_u[col], u1 = s_u[col + 1], u2 = s_u[col + 2], u3 = s_u[col + 3];
#pragma unroll
    for (int p = 0; p < NPASS; ++p) {
        const int r = row0 + p * ROWS_PER_PASS;
        const float kr = s_k[r];
        float4 o4 = make_float4(s[p].x + kr * u0, s[p].y + kr * u1, s[p].z + kr * u2,
                                s[p].w + kr * u3);
        *reinterpret_cast<float4 *>(Sbase + (size_t)r * dv) = o4;
    }
}

// dk = dv = 128: one CTA of 512 threads per (b, h), whole rows per warp.
constexpr int DR_THREADS = 512, DR_D = 128, DR_ROWS = DR_THREADS / 32, DR_NPASS = DR_D / DR_ROWS;

template <typename IO>
__global__ void __launch_bounds__(DR_THREADS, 2)
kda_decode_row_kernel(const IO *__restrict__ q, const IO *__restrict__ k, const IO *__restrict__ v,
                      const IO *__restrict__ g, const IO *__restrict__ beta, float *state,
                      IO *__restrict__ out)
{
    __shared__ float s_alpha[DR_D], s_k[DR_D], s_q[DR_D], s_u[DR_D];
    __shared__ __align__(16) float s_red_a[DR_ROWS][DR_D];
    __shared__ __align__(16) float s_red_b[DR_ROWS][DR_D];
    __shared__ float s_qk;

    const int bh = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t vec = (size_t)bh * DR_D;

    // the state loads go out first, so their latency overlaps the small vector loads below
    const int col4 = lane * 4, row0 = warp;
    float *Sb = state + (size_t)bh * DR_D * DR_D + col4;
    float4 s[DR_NPASS];
#pragma unroll
    for (int p = 0; p < DR_NPASS; ++p) s[p] = *reinterpret_cast<const float4 *>(Sb + (size_t)(row0 + DR_ROWS * p) * DR_D);

    if (tid < DR_D) {
        s_alpha[tid] = __expf(to_f32(g[vec + tid]));
        s_k[tid] = to_f32(k[vec + tid]);
        s_q[tid] = to_f32(q[vec + tid]);
    }
    __syncthreads();
    if (warp == 0) {
        float pq = 0.0f;
        for (int c = lane; c < DR_D; c += 32) pq += s_q[c] * s_k[c];
        pq = warp_sum(pq);
        if (lane == 0) s_qk = pq;
    }
    float a4[4] = {0.f, 0.f, 0.f, 0.f}, b4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int p = 0; p < DR_NPASS; ++p) {
        const int r = row0 + DR_ROWS * p;
        const float al = s_alpha[r], kr = s_k[r], qr = s_q[r];
        s[p].x *= al; s[p].y *= al; s[p].z *= al; s[p].w *= al;
        a4[0] += kr * s[p].x; a4[1] += kr * s[p].y; a4[2] += kr * s[p].z; a4[3] += kr * s[p].w;
        b4[0] += qr * s[p].x; b4[1] += qr * s[p].y; b4[2] += qr * s[p].z; b4[3] += qr * s[p].w;
    }
    *reinterpret_cast<float4 *>(&s_red_a[row0][col4]) = make_float4(a4[0], a4[1], a4[2], a4[3]);
    *reinterpret_cast<float4 *>(&s_red_b[row0][col4]) = make_float4(b4[0], b4[1], b4[2], b4[3]);
    __syncthreads();
    if (tid < DR_D) {
        float sa = 0.f, sb = 0.f;
#pragma unroll
        for (int w = 0; w < DR_ROWS; ++w) {
            sa += s_red_a[w][tid];
            sb += s_red_b[w][tid];
        }
        const float u = to_f32(beta[bh]) * (to_f32(v[vec + tid]) - sa);
        s_u[tid] = u;
        out[vec + tid] = from_f32<IO>(sb + s_qk * u);
    }
    __syncthreads();
    const float u0 = s_u[col4], u1 = s_u[col4 + 1], u2 = s_u[col4 + 2], u3 = s_u[col4 + 3];
#pragma unroll
    for (int p = 0; p < DR_NPASS; ++p) {
        const int r = row0 + DR_ROWS * p;
        const float kr = s_k[r];
        *reinterpret_cast<float4 *>(Sb + (size_t)r * DR_D) =
            make_float4(s[p].x + kr * u0, s[p].y + kr * u1, s[p].z + kr * u2, s[p].w + kr * u3);
    }
}

template <typename IO, int DK>
cudaError_t launch_t(const DecodeArgs &a, cudaStream_t s)
{
    if (DK == DR_D && a.dv == DR_D) {
        kda_decode_row_kernel<IO><<<(unsigned)(a.B * a.H), DR_THREADS, 0, s>>>(
            (const IO *)a.q, (const IO *)a.k, (const IO *)a.v, (const IO *)a.g, (const IO *)a.beta, a.state,
            (IO *)a.out);
        return cudaGetLastError();
    }
    dim3 grid((unsigned)(a.B * a.H), (unsigned)(a.dv / DEC_SLICE));
    kda_decode_kernel<IO, DK><<<grid, DEC_THREADS, 0, s>>>(
        (const IO *)a.q, (const IO *)a.k, (const IO *)a.v, (const IO *)a.g, (const IO *)a.beta,
        a.state, (IO *)a.out, a.H, a.dv);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s)
{
    if (a.io == IO_F32) return a.dk == 64 ? launch_t<float, 64>(a, s) : launch_t<float, 128>(a, s);
    return a.dk == 64 ? launch_t<__nv_bfloat16, 64>(a, s) : launch_t<__nv_bfloat16, 128>(a, s);
}

}  // namespace kda
