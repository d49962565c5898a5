// chunk_f32.cu — exact fp32 chunked prefill on CUDA cores for dk = dv = 128.
//
// It serves the layer path, whose RMSNorm rescales every (token, head) row of o to unit
// RMS so that o must be accurate relative to each row's own RMS (every operand stays
// fp32), and fp32 I/O at d = 128.  One CTA of 256 threads owns one (b, h) and one 64-wide
// half of the value columns and walks the chunks of C = 64 tokens in order.  Within a
// chunk (blocks of 16 tokens; G_i = cumulative log-decay from the chunk start, per channel;
// L_B = block B's log-decay; m_B = its midpoint):
//   E1_i = SC exp(G_i - G_blockstart),  E2_i = SC exp(G_blockend - G_i),  SC = 2^60
//   XQ = q E1,  XK = k E1,  XT = k E2                 (over the loaded q, k, g tiles)
// (the scale keeps E1 and E2 normal numbers for block log-decays down to BAD_LOG, so the
// midpoint factor below never multiplies a flushed zero; every table factor carries 1/SC)
//   P[i,j] = sum_c q_i k_j exp(G_i - G_j)
//          = sum_c (XQ_i fM_B)(XT_j fM_B)   for j in i's block B   (fM_B = exp(-L_B / 2))
//          = sum_c XQ_i XT_j F(J, B)        for j in an earlier block J
//                                            (F = exp of the log-decays of the blocks between)
//   A[i,j] = beta_i (the same with XK_i),  j < i
//   X = Diag(beta) (V - K^ S),   K^ = XK fG  (fG = exp(G_blockstart))
//   U = (I + A)^{-1} X                         (two-level blocked fp32 inverse)
//   O = Q^ S + P U,              Q^ = XQ fG
//   S <- Diag(exp G_C) S + K~^T U,   K~ = XT fL  (fL = exp(G_C - G_blockend))
// Every contraction is a register-tiled fp32 FFMA product out of shared memory.  No
// factor exceeds e^63: a channel whose block log-decay is below BAD_LOG is left out of its
// diagonal block's factorised Gram and that block's terms are added exactly from the raw
// inputs (rare path).  This is the chunkwise form of the gated delta rule of the Kimi
// Delta Attention write-up (the same algebra as the tcgen05 kernel, all in fp32).
#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace kda {
namespace {

constexpr int FNT = 256;     // threads
constexpr int FC = 64;       // chunk
constexpr int FD = 128;      // dk = dv
constexpr int FDH = 64;      // value columns per CTA
constexpr int LDX = FD + 4;  // row stride of the [C][128] tiles (floats)
constexpr int LDH = FDH + 4; // row stride of the [*][64] tiles
constexpr float F32_BAD_LOG = -125.0f;   // SC e^BAD_LOG = e^-83.4 is still a normal number
constexpr float F32_LN_SC = 41.588830f;  // ln SC = 60 ln 2
constexpr float F32_INV_SC = 8.6736174e-19f;  // 2^-60

// shared memory, in floats
constexpr int F_XQ = 0;
constexpr int F_XK = F_XQ + FC * LDX;
constexpr int F_XT = F_XK + FC * LDX;
constexpr int F_V = F_XT + FC * LDX;      // V, then X = Diag(beta)(V - K^ S)
constexpr int F_S = F_V + FC * LDH;       // [128][64] state half
constexpr int F_P = F_S + FD * LDH;
constexpr int F_A = F_P + FC * LDH;       // A, then the inverse's scratch, then U
constexpr int F_LI = F_A + FC * LDH;      // L^{-1}
constexpr int F_TL = F_LI + FC * LDH;     // [4][128] block log-decays L_B
constexpr int F_TG = F_TL + 4 * FD;       // [4][128] fG / SC
constexpr int F_TF = F_TG + 4 * FD;       // [4][128] fL / SC
constexpr int F_TM = F_TF + 4 * FD;       // [4][128] fM / SC (0 where L_B < BAD_LOG)
constexpr int F_TC = F_TM + 4 * FD;       // [3][128] F(0,2), F(0,3), F(1,3), each / SC
constexpr int F_ONE = F_TC + 3 * FD;      // [128] 1 / SC
constexpr int F_GC = F_ONE + FD;          // [128] exp(G_C)
constexpr int F_BETA = F_GC + FD;         // [64]
constexpr int F_MASK = F_BETA + FC;       // uint32 [16]: bad channels per block
constexpr int F_FLOATS = F_MASK + 16;
constexpr size_t F32_SMEM = sizeof(float) * F_FLOATS;
static_assert(F32_SMEM <= 232448, "shared memory per block");
static_assert((F_XK % 4) == 0 && (F_XT % 4) == 0 && (F_V % 4) == 0 && (F_S % 4) == 0 && (F_P % 4) == 0 &&
                  (F_A % 4) == 0 && (F_LI % 4) == 0 && (F_TG % 4) == 0 && (F_TC % 4) == 0 && (F_BETA % 4) == 0,
              "16-byte aligned tiles");

KDA_DEVICE void cp_async16(float *dst, const float *src, bool valid)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(tc::smem_u32(dst)), "l"(src),
                 "r"(valid ? 16 : 0)
                 : "memory");
}
KDA_DEVICE float4 ld4s(const float *p) { return *reinterpret_cast<const float4 *>(p); }
KDA_DEVICE void st4s(float *p, float4 v) { *reinterpret_cast<float4 *>(p) = v; }
KDA_DEVICE float4 mul4(float4 a, float4 b) { return make_float4(a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w); }
KDA_DEVICE float dot4(float4 a, float4 b) { return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w; }
// acc += a.x r0 + a.y r1 + a.z r2 + a.w r3 (component-wise over the float4 rows r)
KDA_DEVICE void axpy4(float4 &acc, float4 a, float4 r0, float4 r1, float4 r2, float4 r3)
{
    acc.x += a.x * r0.x + a.y * r1.x + a.z * r2.x + a.w * r3.x;
    acc.y += a.x * r0.y + a.y * r1.y + a.z * r2.y + a.w * r3.y;
    acc.z += a.x * r0.z + a.y * r1.z + a.z * r2.z + a.w * r3.z;
    acc.w += a.x * r0.w + a.y * r1.w + a.z * r2.w + a.w * r3.w;
}

__global__ void __launch_bounds__(FNT, 1)
kda_chunk_f32_kernel(const float *__restrict__ q, const float *__restrict__ k, const float *__restrict__ v,
                     const float *__restrict__ g, const float *__restrict__ beta, const float *__restrict__ s0,
                     float *__restrict__ out, float *__restrict__ sT, int Ttot, int H, const int *__restrict__ cu)
{
    extern __shared__ __align__(16) float fsm[];
    float *XQ = fsm + F_XQ, *XK = fsm + F_XK, *XT = fsm + F_XT, *Vs = fsm + F_V, *Ss = fsm + F_S;
    float *Ps = fsm + F_P, *As = fsm + F_A, *LI = fsm + F_LI;
    float *TL = fsm + F_TL, *TG = fsm + F_TG, *TF = fsm + F_TF, *TM = fsm + F_TM, *TC = fsm + F_TC;
    float *ONE = fsm + F_ONE, *GCs = fsm + F_GC, *BETAs = fsm + F_BETA;
    uint32_t *MASK = (uint32_t *)(fsm + F_MASK);

    const int tid = threadIdx.x;
    const int bh = blockIdx.x, b = bh / H, h = bh % H;
    const int vh = blockIdx.y;   // value half
    const SeqSpan span = seq_span(cu, b, Ttot);   // this sequence's rows row0 .. row0 + T - 1
    const int T = span.len, row0 = span.row0;
    const size_t soff = (size_t)bh * FD * FD + (size_t)vh * FDH;

    if (tid < FD) ONE[tid] = F32_INV_SC;
    if (tid < 16) MASK[tid] = 0u;
    for (int idx = tid; idx < FD * FDH / 4; idx += FNT) {
        const int c = idx >> 4, j4 = (idx & 15) * 4;
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (s0) x = ld4s(s0 + soff + (size_t)c * FD + j4);
        st4s(Ss + c * LDH + j4, x);
    }

    const int nchunks = (T + FC - 1) / FC;
    for (int n = 0; n < nchunks; ++n) {
        const int t0 = n * FC;
        __syncthreads();   // the previous chunk is fully consumed
        // ------------------------------------------------------------ load (cp.async, zero fill past T)
        for (int idx = tid; idx < FC * FD / 4; idx += FNT) {
            const int i = idx >> 5, c4 = (idx & 31) * 4;
            const bool ok = t0 + i < T;
            const size_t off = ok ? ((size_t)(row0 + t0 + i) * H + h) * FD + c4 : 0;
            cp_async16(XQ + i * LDX + c4, q + off, ok);
            cp_async16(XK + i * LDX + c4, k + off, ok);
            cp_async16(XT + i * LDX + c4, g + off, ok);
        }
        for (int idx = tid; idx < FC * FDH / 4; idx += FNT) {
            const int i = idx >> 4, j4 = (idx & 15) * 4;
            const bool ok = t0 + i < T;
            const size_t off = ok ? ((size_t)(row0 + t0 + i) * H + h) * FD + vh * FDH + j4 : 0;
            cp_async16(Vs + i * LDH + j4, v + off, ok);
        }
        if (tid < FC) BETAs[tid] = t0 + tid < T ? beta[(size_t)(row0 + t0 + tid) * H + h] : 0.0f;
        tc::cp_async_commit();
        tc::cp_async_wait_all();
        __syncthreads();

        // ------------------------------------------------------------ block log-decays
        {
            const int c = tid & (FD - 1), bp = tid >> 7;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int B = 2 * bp + u;
                float acc = 0.0f;
#pragma unroll
                for (int s = 0; s < 16; ++s) acc += XT[(16 * B + s) * LDX + c];
                TL[B * FD + c] = acc;
            }
        }
        __syncthreads();
        // ------------------------------------------------------------ factors and scaled tiles
        {
            const int c = tid & (FD - 1), bp = tid >> 7;
            const float L0 = TL[c], L1 = TL[FD + c], L2 = TL[2 * FD + c], L3 = TL[3 * FD + c];
            if (bp == 0) {
                TC[c] = __expf(L1 - F32_LN_SC);              // F(0, 2) / SC
                TC[FD + c] = __expf(L1 + L2 - F32_LN_SC);    // F(0, 3) / SC
                TC[2 * FD + c] = __expf(L2 - F32_LN_SC);     // F(1, 3) / SC
                GCs[c] = __expf(L0 + L1 + L2 + L3);
            }
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int B = 2 * bp + u;
                const float LB = bp == 0 ? (u == 0 ? L0 : L1) : (u == 0 ? L2 : L3);
                const float lpre = bp == 0 ? (u == 0 ? 0.0f : L0) : (u == 0 ? L0 + L1 : L0 + L1 + L2);
                const float lpost = bp == 0 ? (u == 0 ? L1 + L2 + L3 : L2 + L3) : (u == 0 ? L3 : 0.0f);
                const bool bad = !(LB >= F32_BAD_LOG);
                TG[B * FD + c] = __expf(lpre - F32_LN_SC);
                TF[B * FD + c] = __expf(lpost - F32_LN_SC);
                TM[B * FD + c] = bad ? 0.0f : __expf(-0.5f * LB - F32_LN_SC);
                if (bad) atomicOr(&MASK[B * 4 + (c >> 5)], 1u << (c & 31));
                float G = 0.0f;
#pragma unroll 4
                for (int s = 0; s < 16; ++s) {
                    const int i = 16 * B + s;
                    G += XT[i * LDX + c];
                    const float e1 = __expf(G + F32_LN_SC), e2 = __expf(LB - G + F32_LN_SC);
                    const float kk = XK[i * LDX + c];
                    XQ[i * LDX + c] *= e1;
                    XK[i * LDX + c] = kk * e1;
                    XT[i * LDX + c] = kk * e2;
                }
            }
        }
        __syncthreads();

        // ------------------------------------------------------------ Gram (P, A) and X
        for (int task = tid; task < 576; task += FNT) {
            if (task < 320) {
                // P (m = 0, rows XQ) or A (m = 1, rows XK) for block pair (I, J), J <= I,
                // 4 x 4 outputs: rows 16 I + ti + 4 q, columns 16 J + tj + 4 q'
                const int m = task >= 160;
                const int r = task - 160 * m;
                const int pr = r >> 4, tile = r & 15, ti = tile >> 2, tj = tile & 3;
                const int I = pr < 1 ? 0 : (pr < 3 ? 1 : (pr < 6 ? 2 : 3));
                const int J = pr - I * (I + 1) / 2;
                const float *X = m ? XK : XQ;
                const float *fa = J == I ? TM + I * FD : ONE;
                const float *fb = J == I ? TM + I * FD : (J == I - 1 ? ONE : TC + (J == 0 ? (I == 2 ? 0 : FD) : 2 * FD));
                float acc[4][4];
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[a][e] = 0.0f;
#pragma unroll 2
                for (int c = 0; c < FD; c += 4) {
                    const float4 sa = ld4s(fa + c), sb = ld4s(fb + c);
                    float4 xa[4], xb[4];
#pragma unroll
                    for (int a = 0; a < 4; ++a) {
                        xa[a] = mul4(ld4s(X + (16 * I + ti + 4 * a) * LDX + c), sa);
                        xb[a] = mul4(ld4s(XT + (16 * J + tj + 4 * a) * LDX + c), sb);
                    }
#pragma unroll
                    for (int a = 0; a < 4; ++a)
#pragma unroll
                        for (int e = 0; e < 4; ++e) acc[a][e] += dot4(xa[a], xb[e]);
                }
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    const int i = 16 * I + ti + 4 * a;
                    const float bi = BETAs[i];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = 16 * J + tj + 4 * e;
                        if (m == 0) Ps[i * LDH + j] = j <= i ? acc[a][e] : 0.0f;
                        else As[i * LDH + j] = j < i ? bi * acc[a][e] : 0.0f;
                    }
                }
            } else {
                // X[i, v] = beta_i (V[i, v] - sum_c XK[i, c] fG[c] S[c, v]), rows 4 ti.., columns 4 tj..
                const int x = task - 320, ti = x >> 4, tj = x & 15;
                const float *fg = TG + (ti >> 2) * FD;
                float4 acc[4];
#pragma unroll
                for (int a = 0; a < 4; ++a) acc[a] = ld4s(Vs + (4 * ti + a) * LDH + 4 * tj);
#pragma unroll 2
                for (int c = 0; c < FD; c += 4) {
                    const float4 f = ld4s(fg + c);
                    const float4 s0v = ld4s(Ss + (c + 0) * LDH + 4 * tj), s1v = ld4s(Ss + (c + 1) * LDH + 4 * tj);
                    const float4 s2v = ld4s(Ss + (c + 2) * LDH + 4 * tj), s3v = ld4s(Ss + (c + 3) * LDH + 4 * tj);
#pragma unroll
                    for (int a = 0; a < 4; ++a) {
                        const float4 kh = mul4(ld4s(XK + (4 * ti + a) * LDX + c), f);
                        axpy4(acc[a], make_float4(-kh.x, -kh.y, -kh.z, -kh.w), s0v, s1v, s2v, s3v);
                    }
                }
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    const float bi = BETAs[4 * ti + a];
                    st4s(Vs + (4 * ti + a) * LDH + 4 * tj,
                         make_float4(bi * acc[a].x, bi * acc[a].y, bi * acc[a].z, bi * acc[a].w));
                }
            }
        }
        __syncthreads();

        // ------------------------------------------------------------ exact diagonal blocks of bad channels
        {
            uint32_t any = 0;
#pragma unroll
            for (int w = 0; w < 16; ++w) any |= MASK[w];
            if (any) {
                if (tid < FC) {
                    const int i = tid, I = i >> 4;
                    const float bi = BETAs[i];
                    const bool vi = t0 + i < T;
                    for (int wd = 0; wd < 4; ++wd) {
                        for (uint32_t mk = MASK[I * 4 + wd]; mk != 0u; mk &= mk - 1u) {
                            const int c = 32 * wd + __ffs((int)mk) - 1;
                            const size_t ri = ((size_t)(row0 + t0 + i) * H + h) * FD + c;
                            const float qi = vi ? q[ri] : 0.0f, ki = vi ? k[ri] : 0.0f;
                            float w = 1.0f;   // exp(G_i - G_j), built backwards from j = i
                            for (int j = i; j >= 16 * I; --j) {
                                const bool vj = t0 + j < T;
                                const size_t rj = ((size_t)(row0 + t0 + j) * H + h) * FD + c;
                                const float kj = vj ? k[rj] : 0.0f;
                                Ps[i * LDH + j] += qi * kj * w;
                                if (j < i) As[i * LDH + j] += bi * ki * kj * w;
                                w *= __expf(vj ? g[rj] : 0.0f);
                            }
                        }
                    }
                }
                __syncthreads();
            }
        }
        if (tid < 16) MASK[tid] = 0u;   // read above by every thread before the barrier

        // ------------------------------------------------------------ L^{-1}, L = I + A
        // 16x16 diagonal inverses (right-looking substitution), then the 2x2 block rule
        // [[L_a, 0], [A_ba, L_b]]^{-1} = [[L_a^{-1}, 0], [-L_b^{-1} A_ba L_a^{-1}, L_b^{-1}]]
        // for the 32x32 halves and once more for the whole 64x64.
        if (tid < FC) {
            const int Ib = tid >> 4, col = tid & 15;
            float x[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) x[r] = r == col ? 1.0f : 0.0f;
#pragma unroll
            for (int m = 0; m < 15; ++m)
#pragma unroll
                for (int r = m + 1; r < 16; ++r) x[r] -= As[(16 * Ib + r) * LDH + 16 * Ib + m] * x[m];
#pragma unroll
            for (int r = 0; r < 16; ++r) LI[(16 * Ib + r) * LDH + 16 * Ib + col] = x[r];
        }
        __syncthreads();
        auto dot16 = [&](const float *Xm, int xr, int xc, const float *Ym, int yr, int yc) -> float {
            float s0a = 0.0f, s1a = 0.0f;
#pragma unroll
            for (int m4 = 0; m4 < 16; m4 += 4) {
                const float4 xv = ld4s(Xm + xr * LDH + xc + m4);
                s0a += xv.x * Ym[(yr + m4) * LDH + yc] + xv.z * Ym[(yr + m4 + 2) * LDH + yc];
                s1a += xv.y * Ym[(yr + m4 + 1) * LDH + yc] + xv.w * Ym[(yr + m4 + 3) * LDH + yc];
            }
            return s0a + s1a;
        };
        {
            const int r = tid >> 4, c = tid & 15;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
                As[r * LDH + 32 + 16 * hh + c] = dot16(As, 32 * hh + 16 + r, 32 * hh, LI, 32 * hh, 32 * hh + c);
            __syncthreads();
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int ra = 32 * hh, rb = ra + 16;
                LI[(rb + r) * LDH + ra + c] = -dot16(LI, rb + r, rb, As, 0, 32 + 16 * hh + c);
                LI[(ra + r) * LDH + rb + c] = 0.0f;
            }
            __syncthreads();
        }
        {
            // Q = A_{[2,3],[0,1]} L_{[0,1]}^{-1} -> A's upper-right 32x32; then
            // L^{-1}_{[2,3],[0,1]} = -L_{[2,3]}^{-1} Q.  4 rows x 1 column per thread.
            const int c = tid & 31, rg = tid >> 5;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int m4 = 0; m4 < 32; m4 += 4) {
                float y[4];
#pragma unroll
                for (int t = 0; t < 4; ++t) y[t] = LI[(m4 + t) * LDH + c];
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    const float4 xv = ld4s(As + (32 + 4 * rg + a) * LDH + m4);
                    acc[a] += xv.x * y[0] + xv.y * y[1] + xv.z * y[2] + xv.w * y[3];
                }
            }
#pragma unroll
            for (int a = 0; a < 4; ++a) As[(4 * rg + a) * LDH + 32 + c] = acc[a];
            __syncthreads();
#pragma unroll
            for (int a = 0; a < 4; ++a) acc[a] = 0.0f;
#pragma unroll
            for (int m4 = 0; m4 < 32; m4 += 4) {
                float y[4];
#pragma unroll
                for (int t = 0; t < 4; ++t) y[t] = As[(m4 + t) * LDH + 32 + c];
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    const float4 xv = ld4s(LI + (32 + 4 * rg + a) * LDH + 32 + m4);
                    acc[a] += xv.x * y[0] + xv.y * y[1] + xv.z * y[2] + xv.w * y[3];
                }
            }
#pragma unroll
            for (int a = 0; a < 4; ++a) LI[(32 + 4 * rg + a) * LDH + c] = -acc[a];
            __syncthreads();
        }

        // ------------------------------------------------------------ U = L^{-1} X  (into A's tile)
        const int ti = tid >> 4, tj = tid & 15;
        {
            float4 acc[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) acc[a] = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int j = 0; j <= 4 * ti; j += 4) {
                const float4 x0 = ld4s(Vs + (j + 0) * LDH + 4 * tj), x1 = ld4s(Vs + (j + 1) * LDH + 4 * tj);
                const float4 x2 = ld4s(Vs + (j + 2) * LDH + 4 * tj), x3 = ld4s(Vs + (j + 3) * LDH + 4 * tj);
#pragma unroll
                for (int a = 0; a < 4; ++a) axpy4(acc[a], ld4s(LI + (4 * ti + a) * LDH + j), x0, x1, x2, x3);
            }
#pragma unroll
            for (int a = 0; a < 4; ++a) st4s(As + (4 * ti + a) * LDH + 4 * tj, acc[a]);
        }
        __syncthreads();
        // ------------------------------------------------------------ O = Q^ S + P U
        {
            const float *fg = TG + (ti >> 2) * FD;
            float4 acc[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) acc[a] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
            for (int c = 0; c < FD; c += 4) {
                const float4 f = ld4s(fg + c);
                const float4 s0v = ld4s(Ss + (c + 0) * LDH + 4 * tj), s1v = ld4s(Ss + (c + 1) * LDH + 4 * tj);
                const float4 s2v = ld4s(Ss + (c + 2) * LDH + 4 * tj), s3v = ld4s(Ss + (c + 3) * LDH + 4 * tj);
#pragma unroll
                for (int a = 0; a < 4; ++a) axpy4(acc[a], mul4(ld4s(XQ + (4 * ti + a) * LDX + c), f), s0v, s1v, s2v, s3v);
            }
            for (int j = 0; j <= 4 * ti; j += 4) {
                const float4 u0 = ld4s(As + (j + 0) * LDH + 4 * tj), u1 = ld4s(As + (j + 1) * LDH + 4 * tj);
                const float4 u2 = ld4s(As + (j + 2) * LDH + 4 * tj), u3 = ld4s(As + (j + 3) * LDH + 4 * tj);
#pragma unroll
                for (int a = 0; a < 4; ++a) axpy4(acc[a], ld4s(Ps + (4 * ti + a) * LDH + j), u0, u1, u2, u3);
            }
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int i = 4 * ti + a;
                if (t0 + i < T) st4s(out + ((size_t)(row0 + t0 + i) * H + h) * FD + vh * FDH + 4 * tj, acc[a]);
            }
        }
        __syncthreads();
        // ------------------------------------------------------------ S <- Diag(exp G_C) S + K~^T U
        {
            // rows c = 8 ti .. 8 ti + 7, columns 4 tj ..
            float4 acc[8];
#pragma unroll
            for (int a = 0; a < 8; ++a) {
                const float gc = GCs[8 * ti + a];
                const float4 sv = ld4s(Ss + (8 * ti + a) * LDH + 4 * tj);
                acc[a] = make_float4(gc * sv.x, gc * sv.y, gc * sv.z, gc * sv.w);
            }
            for (int i = 0; i < FC; i += 4) {
                const float *fl = TF + (i >> 4) * FD + 8 * ti;
                const float4 fl0 = ld4s(fl), fl1 = ld4s(fl + 4);
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const float4 kt0 = mul4(ld4s(XT + (i + t) * LDX + 8 * ti), fl0);
                    const float4 kt1 = mul4(ld4s(XT + (i + t) * LDX + 8 * ti + 4), fl1);
                    const float4 u = ld4s(As + (i + t) * LDH + 4 * tj);
                    const float kv[8] = {kt0.x, kt0.y, kt0.z, kt0.w, kt1.x, kt1.y, kt1.z, kt1.w};
#pragma unroll
                    for (int a = 0; a < 8; ++a) {
                        acc[a].x += kv[a] * u.x;
                        acc[a].y += kv[a] * u.y;
                        acc[a].z += kv[a] * u.z;
                        acc[a].w += kv[a] * u.w;
                    }
                }
            }
#pragma unroll
            for (int a = 0; a < 8; ++a) st4s(Ss + (8 * ti + a) * LDH + 4 * tj, acc[a]);
        }
    }
    __syncthreads();
    if (sT) {
        for (int idx = tid; idx < FD * FDH / 4; idx += FNT) {
            const int c = idx >> 4, j4 = (idx & 15) * 4;
            st4s(sT + soff + (size_t)c * FD + j4, ld4s(Ss + c * LDH + j4));
        }
    }
}

}  // namespace

bool chunk_f32_supported(const ChunkArgs &a)
{
    const bool all_f32 = a.io == IO_F32 || (a.qkv_f32 && a.g_f32 && a.beta_f32 && a.out_f32);
    return all_f32 && a.dk == FD && a.dv == FD && a.T > 0;
}

cudaError_t launch_chunk_f32(const ChunkArgs &a, cudaStream_t s)
{
    struct Tag;
    const cudaError_t attr = smem_opt_in<Tag>((const void *)kda_chunk_f32_kernel, (int)F32_SMEM);
    if (attr != cudaSuccess) return attr;
    dim3 grid((unsigned)(a.B * a.H), 2u);
    kda_chunk_f32_kernel<<<grid, FNT, F32_SMEM, s>>>((const float *)a.q, (const float *)a.k, (const float *)a.v,
                                                     (const float *)a.g, (const float *)a.beta, a.s0,
                                                     (float *)a.out, a.sT, a.T, a.H, a.cu);
    return cudaGetLastError();
}

}  // namespace kda
