// chunk_simt.cu — chunkwise KDA prefill on CUDA cores (fp32 FFMA throughout).
//
// This is the exact path: it serves fp32 I/O (where the parity bar is 1e-4 of the
// output's max) and the d = 64 shapes.  bf16 I/O at d = 128 runs on the tcgen05
// kernel instead (chunk_tc.cu).
//
// Chunkwise form of the gated delta rule (per head, chunk of C = 64 tokens, chunk
// start state S0, cumulative per-channel log-decay G_i = sum_{s<=i} g_s):
//     A[i,j] = beta_i sum_c k_i[c] k_j[c] exp(G_i[c] - G_j[c])       (j < i)
//     P[i,j] =        sum_c q_i[c] k_j[c] exp(G_i[c] - G_j[c])       (j <= i)
//     (I + A) U = Diag(beta) (V - (exp(G) * K) S0)                   (forward substitution)
//     O   = (exp(G) * Q) S0 + P U
//     S_C = Diag(exp G_C) S0 + (exp(G_C - G) * K)^T U
// Every exponent above is <= 0, so no factor can overflow; the pairwise factors
// are formed directly on the MUFU.  One CTA owns one (b, h) and one 64-wide slice
// of the value columns (columns are independent), and walks the chunks in order.
// Rows past the end of the sequence are zero-filled with g = 0, beta = 0, so they
// neither decay nor write the state.
#include "common.cuh"
#include "internal.h"

namespace kda {
namespace {

constexpr int CS_THREADS = 256;
constexpr int CS_C = 64;    // chunk length
constexpr int CS_DVS = 64;  // value columns per CTA

template <int DK>
struct SimtSmem {
    static constexpr int LDK = DK + 1;          // padded row stride of the [C, DK] tiles
    static constexpr int LDV = CS_DVS + 1;      // padded row stride of [*, 64] tiles
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + CS_C * LDK;
    static constexpr int OFF_G = OFF_K + CS_C * LDK;
    static constexpr int OFF_U = OFF_G + CS_C * LDK;     // V, then RHS, then U
    static constexpr int OFF_S = OFF_U + CS_C * LDV;     // [DK, 64] state slice
    static constexpr int OFF_P = OFF_S + DK * LDV;
    static constexpr int OFF_A = OFF_P + CS_C * LDV;
    static constexpr int OFF_B = OFF_A + CS_C * LDV;     // beta [C]
    static constexpr int OFF_GC = OFF_B + CS_C;          // G_C [DK]
    static constexpr int FLOATS = OFF_GC + DK;
    static constexpr size_t BYTES = sizeof(float) * FLOATS;
};

template <typename TI, typename TG, typename TB, typename TO, int DK>
__global__ void __launch_bounds__(CS_THREADS, 1)
kda_chunk_simt_kernel(const TI *__restrict__ q, const TI *__restrict__ k, const TI *__restrict__ v,
                      const TG *__restrict__ g, const TB *__restrict__ beta,
                      const float *__restrict__ s0, TO *__restrict__ out, float *__restrict__ sT,
                      int Ttot, int H, int dv, const int *__restrict__ cu)
{
    using L = SimtSmem<DK>;
    extern __shared__ float smem[];
    float *Qs = smem + L::OFF_Q, *Ks = smem + L::OFF_K, *Gs = smem + L::OFF_G;
    float *Us = smem + L::OFF_U, *Ss = smem + L::OFF_S, *Ps = smem + L::OFF_P;
    float *As = smem + L::OFF_A, *Bs = smem + L::OFF_B, *GCs = smem + L::OFF_GC;

    const int tid = threadIdx.x;
    const int bh = blockIdx.x;
    const int b = bh / H, h = bh % H;
    const int v0 = blockIdx.y * CS_DVS;
    const SeqSpan span = seq_span(cu, b, Ttot);   // this sequence's rows row0 .. row0 + T - 1
    const int T = span.len, row0 = span.row0;
    const size_t state_off = (size_t)bh * DK * dv + v0;

    // initial state slice
    for (int idx = tid; idx < DK * CS_DVS; idx += CS_THREADS) {
        const int c = idx / CS_DVS, j = idx % CS_DVS;
        Ss[c * L::LDV + j] = s0 ? s0[state_off + (size_t)c * dv + j] : 0.0f;
    }

    const int nchunks = (T + CS_C - 1) / CS_C;
    for (int n = 0; n < nchunks; ++n) {
        const int t0 = n * CS_C;
        const int nt = min(CS_C, T - t0);
        __syncthreads();  // previous chunk fully consumed
        // ---------------------------------------------------------------- load
        for (int idx = tid; idx < CS_C * DK / 4; idx += CS_THREADS) {
            const int i = idx / (DK / 4), c = (idx % (DK / 4)) * 4;
            float fq[4] = {0.f, 0.f, 0.f, 0.f}, fk[4] = {0.f, 0.f, 0.f, 0.f},
                  fg[4] = {0.f, 0.f, 0.f, 0.f};
            if (i < nt) {
                const size_t off = ((size_t)(row0 + t0 + i) * H + h) * DK + c;
                ld4(q + off, fq);
                ld4(k + off, fk);
                ld4(g + off, fg);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                Qs[i * L::LDK + c + e] = fq[e];
                Ks[i * L::LDK + c + e] = fk[e];
                Gs[i * L::LDK + c + e] = fg[e];
            }
        }
        for (int idx = tid; idx < CS_C * CS_DVS / 4; idx += CS_THREADS) {
            const int i = idx / (CS_DVS / 4), j = (idx % (CS_DVS / 4)) * 4;
            float fv[4] = {0.f, 0.f, 0.f, 0.f};
            if (i < nt) ld4(v + ((size_t)(row0 + t0 + i) * H + h) * dv + v0 + j, fv);
#pragma unroll
            for (int e = 0; e < 4; ++e) Us[i * L::LDV + j + e] = fv[e];
        }
        if (tid < CS_C) Bs[tid] = tid < nt ? to_f32(beta[(size_t)(row0 + t0 + tid) * H + h]) : 0.0f;
        __syncthreads();
        // ---------------------------------------------------------------- G = cumsum(g)
        if (tid < DK) {
            float acc = 0.0f;
            for (int i = 0; i < CS_C; ++i) {
                acc += Gs[i * L::LDK + tid];
                Gs[i * L::LDK + tid] = acc;
            }
            GCs[tid] = acc;
        }
        __syncthreads();
        // ---------------------------------------------------------------- Gram P, A and RHS
        {
            const int i = tid >> 2, part = tid & 3;
            float p[16], a[16];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) { p[jj] = 0.f; a[jj] = 0.f; }
            for (int c = 0; c < DK; ++c) {
                const float qi = Qs[i * L::LDK + c], ki = Ks[i * L::LDK + c], gi = Gs[i * L::LDK + c];
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) {
                    const int j = part + 4 * jj;
                    if (j <= i) {
                        const float kj = Ks[j * L::LDK + c];
                        const float w = __expf(gi - Gs[j * L::LDK + c]) * kj;
                        p[jj] += qi * w;
                        a[jj] += ki * w;
                    }
                }
            }
            const float bi = Bs[i];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
                const int j = part + 4 * jj;
                Ps[i * L::LDV + j] = j <= i ? p[jj] : 0.0f;
                As[i * L::LDV + j] = j < i ? bi * a[jj] : 0.0f;
            }
            // RHS[i, v] = beta_i (V[i, v] - sum_c exp(G_i[c]) K[i, c] S[c, v]), in place over V
            float r[16];
#pragma unroll
            for (int vv = 0; vv < 16; ++vv) r[vv] = 0.f;
            for (int c = 0; c < DK; ++c) {
                const float kh = Ks[i * L::LDK + c] * __expf(Gs[i * L::LDK + c]);
#pragma unroll
                for (int vv = 0; vv < 16; ++vv) r[vv] += kh * Ss[c * L::LDV + part + 4 * vv];
            }
#pragma unroll
            for (int vv = 0; vv < 16; ++vv) {
                float *u = &Us[i * L::LDV + part + 4 * vv];
                *u = bi * (*u - r[vv]);
            }
        }
        __syncthreads();
        // ---------------------------------------------------------------- forward substitution
        {
            // warp w owns value columns 8w..8w+7; 4 lanes per column split the j sum
            const int col = tid >> 2, part = tid & 3;
            for (int i = 1; i < CS_C; ++i) {
                float s = 0.0f;
                for (int j = part; j < i; j += 4) s += As[i * L::LDV + j] * Us[j * L::LDV + col];
                s += __shfl_xor_sync(0xffffffffu, s, 1);
                s += __shfl_xor_sync(0xffffffffu, s, 2);
                if (part == 0) Us[i * L::LDV + col] -= s;
                __syncwarp();
            }
        }
        __syncthreads();
        // ---------------------------------------------------------------- O = (e^G Q) S0 + P U
        {
            const int i = tid >> 2, part = tid & 3;
            float o[16];
#pragma unroll
            for (int vv = 0; vv < 16; ++vv) o[vv] = 0.f;
            for (int c = 0; c < DK; ++c) {
                const float qh = Qs[i * L::LDK + c] * __expf(Gs[i * L::LDK + c]);
#pragma unroll
                for (int vv = 0; vv < 16; ++vv) o[vv] += qh * Ss[c * L::LDV + part + 4 * vv];
            }
            for (int j = 0; j <= i; ++j) {
                const float pij = Ps[i * L::LDV + j];
#pragma unroll
                for (int vv = 0; vv < 16; ++vv) o[vv] += pij * Us[j * L::LDV + part + 4 * vv];
            }
            if (i < nt) {
                TO *orow = out + ((size_t)(row0 + t0 + i) * H + h) * dv + v0;
#pragma unroll
                for (int vv = 0; vv < 16; ++vv) orow[part + 4 * vv] = from_f32<TO>(o[vv]);
            }
        }
        __syncthreads();
        // ---------------------------------------------------------------- S <- e^{G_C} S + (e^{G_C - G} K)^T U
        {
            constexpr int TPC = CS_THREADS / DK;     // threads per key channel: 2 or 4
            constexpr int NV = CS_DVS / TPC;         // columns per thread
            const int c = tid / TPC, part = tid % TPC;
            const float gc = GCs[c];
            const float dc = __expf(gc);
            float acc[NV];
#pragma unroll
            for (int vv = 0; vv < NV; ++vv) acc[vv] = dc * Ss[c * L::LDV + part + TPC * vv];
            for (int i = 0; i < CS_C; ++i) {
                const float kt = Ks[i * L::LDK + c] * __expf(gc - Gs[i * L::LDK + c]);
#pragma unroll
                for (int vv = 0; vv < NV; ++vv) acc[vv] += kt * Us[i * L::LDV + part + TPC * vv];
            }
#pragma unroll
            for (int vv = 0; vv < NV; ++vv) Ss[c * L::LDV + part + TPC * vv] = acc[vv];
        }
    }
    __syncthreads();
    if (sT) {
        for (int idx = tid; idx < DK * CS_DVS; idx += CS_THREADS) {
            const int c = idx / CS_DVS, j = idx % CS_DVS;
            sT[state_off + (size_t)c * dv + j] = Ss[c * L::LDV + j];
        }
    }
}

template <typename TI, typename TG, typename TB, typename TO, int DK>
cudaError_t launch_t(const ChunkArgs &a, cudaStream_t s)
{
    auto kern = kda_chunk_simt_kernel<TI, TG, TB, TO, DK>;
    const size_t bytes = SimtSmem<DK>::BYTES;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)(a.B * a.H), (unsigned)(a.dv / CS_DVS));
    kern<<<grid, CS_THREADS, bytes, s>>>((const TI *)a.q, (const TI *)a.k, (const TI *)a.v,
                                          (const TG *)a.g, (const TB *)a.beta, a.s0, (TO *)a.out,
                                          a.sT, a.T, a.H, a.dv, a.cu);
    return cudaGetLastError();
}

template <typename TI, typename TG, typename TB, typename TO>
cudaError_t launch_dk(const ChunkArgs &a, cudaStream_t s)
{
    return a.dk == 64 ? launch_t<TI, TG, TB, TO, 64>(a, s) : launch_t<TI, TG, TB, TO, 128>(a, s);
}

}  // namespace

cudaError_t launch_chunk_simt(const ChunkArgs &a, cudaStream_t s)
{
    using bf = __nv_bfloat16;
    // all-fp32 operands: the fp32 I/O path and the layer path's fp32 workspace
    if (a.io == IO_F32 || (a.qkv_f32 && a.g_f32 && a.beta_f32 && a.out_f32))
        return launch_dk<float, float, float, float>(a, s);
    return launch_dk<bf, bf, bf, bf>(a, s);
}

}  // namespace kda
