// chunk_tc.cu — chunked KDA prefill on tcgen05 tensor cores (bf16 I/O, dk = dv = 128).
//
// One CTA owns one (b, h) head and walks its chunks of C = 64 tokens in order.  The
// fp32 state lives in tensor memory for the whole sequence, transposed (lane = value
// column v, column = key channel c), next to its bf16 copy that feeds the MMAs as
// the A operand.  Per chunk, with G_i = sum_{s<=i} g_s (per channel) and blocks of 16
// tokens inside the chunk:
//
//   prep (CUDA cores)   alpha = exp(g); in-block prefix/suffix products give
//                       e1_i = exp(G_i - G_start(blk)), e2_i = exp(G_end(blk) - G_i) and the
//                       block decays D_B; from them Q^ = Gamma*Q, K^ = Gamma*K,
//                       K~ = exp(G_C - G)*K and the Gram operands (below).
//   Gram (tcgen05)      [Q;K] rows x CV_I columns -> P (j <= i) and A' (j < i) in one
//                       M=128, N=160, K=128 MMA.
//   inverse (CUDA)      T = (I + Diag(beta) A')^{-1} Diag(beta), blocked by 16, fp32.
//   W, U~ (tcgen05)     W^T = K^^T T^T, U~^T = V^T T^T.
//   chain (tcgen05)     U^T = U~^T - S^T W^T;  O^T = S^T Q^^T + U^T P^T;
//                       S^T <- S^T Diag(exp G_C) + U^T K~.
// The two products that read the state (S^T Q^^T and S^T W^T) run as kind::tf32 MMAs
// with the fp32 state itself, straight from tensor memory, as the A operand.
//
// Overflow-safe Gram factorisation.  exp(G_i - G_j) (j <= i) spans far more than the
// fp32 range over a chunk, so it is never formed as exp(G_i) exp(-G_j).  Row i of
// block I is scaled by exp(G_i - m_I), m_I the midpoint of block I's log-decay range,
// and the column operand used by block I's rows is
//     CV_I[j] = k_j exp(m_I - G_j)   for every j in blocks 0..I,
// so every pair (i in block I, j <= i) gets exactly exp(G_i - G_j).  Off-diagonal
// factors are products of in-block decays (all <= 1); only the diagonal block carries
// factors up to exp(range_I / 2).  A channel whose decay over block I exceeds e^168
// ("bad") falls back to the block-start reference for its rows, is left out of
// block I's diagonal in the MMA, and has that diagonal added exactly on CUDA cores.
//
// Precision.  bf16 operands alone would put errors of the order of one bf16 rounding
// on top of the output's own bf16 rounding.  So the diagonal P[i][i] = q_i . k_i is
// formed exactly in fp32 from the raw inputs, the diagonal 16x16 blocks of the Gram get a
// second MMA with the rounding residuals (R_lo CVd + R CVd_lo), U and P enter their products as
// hi + lo bf16 pairs (O += U_hi P_hi + U_lo P_hi + U_hi P_lo, S += K~^T (U_hi + U_lo)),
// and the state is read at tf32 precision from its fp32 copy (Q^ and W kept in fp32).
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace kda {
namespace {

using namespace tc;

constexpr int NT = 256;       // threads
constexpr int CK = 64;        // chunk
constexpr int DD = 128;       // dk = dv
constexpr float BAD_LOG = -168.0f;  // block log-decays below this take the exact fallback

// shared memory layout (offsets from a 1024-byte aligned base)
constexpr int REG_BYTES = 73728;                 // 72 KB: stage (q,k,v,g) or Gram operands
constexpr int OFF_REG0 = 0;
constexpr int OFF_REG1 = REG_BYTES;
constexpr int ST_Q = 0, ST_K = 16384, ST_V = 32768, ST_G = 49152;     // inside a stage region
constexpr int GR_R = 0, GR_CV = 32768;                                // inside a Gram region
constexpr int R_CB = 16384;                      // R: 128 rows x 128 B per channel block
constexpr int CV_ROWS = 160, CV_CB = CV_ROWS * 128;
// X1 (32 KB): Q^ in fp32 (tf32 K-major [i][c], prep -> O init); then P, P_lo, T (bf16)
// X2 (32 KB): A and L^{-1} in fp32 (inverse); then W in fp32 (tf32 K-major [i][c])
constexpr int OFF_X1 = 2 * REG_BYTES;
constexpr int OFF_QH = OFF_X1;                   // 32 KB: 4 K-blocks of 32 fp32 x 64 rows
constexpr int OFF_P = OFF_X1;                    // 8 KB bf16 K-major [i][j]: P (hi part)
constexpr int OFF_PL = OFF_P + 8192;             // 8 KB bf16: P - P_hi (lo part)
constexpr int OFF_T = OFF_PL + 8192;             // 8 KB bf16 K-major [i][j]
constexpr int OFF_X2 = OFF_X1 + 32768;
constexpr int OFF_A32 = OFF_X2;                  // 16 KB fp32 [64][64]
constexpr int OFF_LINV = OFF_X2 + 16384;         // 16 KB fp32 [64][64]
constexpr int OFF_W = OFF_X2;                    // 32 KB: 4 K-blocks of 32 fp32 x 64 rows
constexpr int OFF_MISC = OFF_X2 + 32768;
constexpr int MS_BADMASK = 0;                    // uint32 [4][4]: channels with L_B < BAD_LOG, per block
constexpr int MS_GC = 2048;                      // fp32 [128] chunk decay exp(G_C)
constexpr int MS_BETA = 2560;                    // fp32 [64]
constexpr int MS_PD = 3344;                      // fp32 [2][64]: exact q_i . k_i halves
constexpr int MS_BAR = 3856;                     // uint64 [3]: tma0, tma1, mma
constexpr int MS_TSLOT = 3880;                   // uint32
constexpr int MS_ABORT = 3884;                   // int
constexpr int MISC_BYTES = 3904;
// per-(block, channel) factor table, fp32 [slot][128]: fG, fL, fM, fD for blocks 0..3, then
// fC for the six (B, I) pairs with I > B
constexpr int FT_G = 0, FT_L = 4 * 128, FT_M = 8 * 128, FT_D = 12 * 128, FT_C = 16 * 128;
constexpr int FT_BYTES = 22 * 128 * 4;
constexpr int OFF_FT = OFF_MISC + MISC_BYTES;
constexpr int SMEM_BYTES = OFF_FT + FT_BYTES + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory per block");
__host__ __device__ constexpr int fc_slot(int B, int I) { return B == 0 ? I - 1 : (B == 1 ? I + 1 : 5); }

// tensor memory columns
constexpr uint32_t TM_S = 0;     // fp32 S^T, 128 cols
constexpr uint32_t TM_G = 128;   // Gram D, 160 cols (W^T reuses the first 64)
constexpr uint32_t TM_W = 128;
constexpr uint32_t TM_UL = 192;  // bf16 (U - U_hi)^T (A operand), 32 cols, inside the Gram area
constexpr uint32_t TM_U = 288;   // U^T, 64 cols
constexpr uint32_t TM_O = 352;   // O^T, 64 cols
constexpr uint32_t TM_CORR = 416;  // diagonal-block Gram correction R_lo CVd + R CVd_lo, 64 cols
constexpr uint32_t TM_UB = 480;  // bf16 U^T (A operand), 32 cols

// Gram column buffer: rows 0..63 are the diagonal-block columns (row j for token j);
// rows cv_off(I) + j (j < 16 I) are block I's columns for earlier tokens.
__host__ __device__ constexpr int cv_off(int I) { return I == 1 ? 64 : I == 2 ? 80 : 112; }

struct TcParams {
    const __nv_bfloat16 *q, *k, *g, *beta;
    const float *s0;
    __nv_bfloat16 *out;
    float *sT;
    int T, H;
    int *err;
};

KDA_DEVICE void unpack8(const uint4 &u, float (&f)[8])
{
    float2 a = unpack_bf16x2(u.x), b = unpack_bf16x2(u.y), c = unpack_bf16x2(u.z), d = unpack_bf16x2(u.w);
    f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y; f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}
KDA_DEVICE uint4 pack8(const float (&f)[8])
{
    return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                      pack_bf16x2(f[6], f[7]));
}

__global__ void __launch_bounds__(NT, 1)
kda_chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                    const __grid_constant__ CUtensorMap tm_o, TcParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *misc = sm + OFF_MISC;
    uint32_t *badmask = (uint32_t *)(misc + MS_BADMASK);
    float *FT = (float *)(sm + OFF_FT);
    float *PDsm = (float *)(misc + MS_PD);
    float *GCsm = (float *)(misc + MS_GC);
    float *BETAsm = (float *)(misc + MS_BETA);
    uint64_t *bar_tma = (uint64_t *)(misc + MS_BAR);
    uint64_t *bar_mma = bar_tma + 2;
    uint32_t *tslot = (uint32_t *)(misc + MS_TSLOT);
    volatile int *abort_flag = (volatile int *)(misc + MS_ABORT);
    float *A32 = (float *)(sm + OFF_A32);
    float *LINV = (float *)(sm + OFF_LINV);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x, b = bh / p.H, h = bh % p.H;
    const int T = p.T;
    const int nchunks = (T + CK - 1) / CK;
    const uint32_t lane_q = (uint32_t)(32 * (warp & 3)) << 16;   // this warp's TMEM lane quarter
    const int half = warp >> 2;

    if (tid == 0) {
        mbar_init(&bar_tma[0], 1);
        mbar_init(&bar_tma[1], 1);
        mbar_init(bar_mma, 1);
        *abort_flag = 0;
        for (int i = 0; i < 16; ++i) badmask[i] = 0u;
        fence_mbar_init();
        prefetch_tmap(&tm_q); prefetch_tmap(&tm_k); prefetch_tmap(&tm_v); prefetch_tmap(&tm_g);
        prefetch_tmap(&tm_o);
    }
    if (warp == 0) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;

    auto issue_tma = [&](int n) {
        const int r = n & 1;
        uint8_t *st = sm + (r ? OFF_REG1 : OFF_REG0);
        const int t0 = n * CK;
        mbar_arrive_expect_tx(&bar_tma[r], 4 * 16384);
        for (int cb = 0; cb < 2; ++cb) {
            tma_load_4d(st + ST_Q + cb * 8192, &tm_q, cb * 64, h, t0, b, &bar_tma[r]);
            tma_load_4d(st + ST_K + cb * 8192, &tm_k, cb * 64, h, t0, b, &bar_tma[r]);
            tma_load_4d(st + ST_V + cb * 8192, &tm_v, cb * 64, h, t0, b, &bar_tma[r]);
            tma_load_4d(st + ST_G + cb * 8192, &tm_g, cb * 64, h, t0, b, &bar_tma[r]);
        }
    };
    if (tid == 0 && nchunks > 0) issue_tma(0);

    // ---------------------------------------------------------------- initial state
    {
        const int v = 32 * (warp & 3) + lane;
        const float *s0 = p.s0 ? p.s0 + (size_t)bh * DD * DD : nullptr;
        for (int cc = 0; cc < 64; cc += 32) {
            uint32_t r[32];
            for (int e = 0; e < 32; ++e) {
                const int c = 64 * half + cc + e;
                r[e] = __float_as_uint(s0 ? s0[(size_t)c * DD + v] : 0.0f);
            }
            tmem_st32(tmem + lane_q + TM_S + 64 * half + cc, r);
        }
        tmem_wait_st();
    }

    uint32_t mma_phase = 0;
    auto mma_wait = [&]() -> bool {
        const bool ok = mbar_wait_bounded(bar_mma, mma_phase, abort_flag, p.err);
        mma_phase ^= 1u;
        return ok;
    };

    const uint32_t id_gram = idesc_bf16(128, CV_ROWS, false, false);
    const uint32_t id_corr = idesc_bf16(128, 64, false, false);
    const uint32_t id_o0 = idesc_tf32(128, 64, false, false);
    const uint32_t id_wt = idesc_bf16(128, 64, true, false);
    const uint32_t id_u = idesc_tf32(128, 64, false, false, true);
    const uint32_t id_op = idesc_bf16(128, 64, false, false);
    const uint32_t id_s = idesc_bf16(128, 128, false, true);

    // beta of the next chunk is loaded one chunk ahead, so its global-memory latency never
    // sits on the path into prep
    auto load_beta = [&](int n) -> float {
        const int t = n * CK + tid;
        return (tid < CK && t < T) ? __bfloat162float(p.beta[(size_t)(b * T + t) * p.H + h]) : 0.0f;
    };
    float beta_next = nchunks > 0 ? load_beta(0) : 0.0f;

    for (int n = 0; n < nchunks; ++n) {
        const int X = n & 1;
        uint8_t *stg = sm + (X ? OFF_REG1 : OFF_REG0);
        uint8_t *gro = sm + (X ? OFF_REG0 : OFF_REG1);
        const int t0 = n * CK;
        const int nt = min(CK, T - t0);

        // the previous chunk's O tile must have left X2 before this chunk writes there (after
        // the barrier inside prep)
        if (tid == 0) bulk_wait_read_all();
        if (!mbar_wait_bounded(&bar_tma[X], (uint32_t)((n >> 1) & 1), abort_flag, p.err)) break;

        // ============================================================ prep
        if (tid < CK) BETAsm[tid] = beta_next;
        beta_next = n + 1 < nchunks ? load_beta(n + 1) : 0.0f;
        constexpr float INV_SC = 7.523164e-37f;    // SC = 2^120, INV_SC = 2^-120
        constexpr float LN_SC = 83.17766f;         // 120 ln 2
        // pass 1: block log-decays L_B (sum of g over a 16-token block) per channel, and from
        // them the per-(block, channel) factor table, computed once per chunk:
        //   fG = exp(G_blockstart)      fL = exp(G_C - G_blockend)
        //   fM = exp(-L_B / 2) / SC     (block-start reference, 1 / SC, where L_B < BAD_LOG)
        //   fD = fM, or 0 where L_B < BAD_LOG (those diagonal terms are added exactly later)
        //   fC(B, I) = exp(m_I - G_blockend of B) for later blocks I > B, m_I the reference of I
        // All exponents are sums of non-positive log-decays (plus L_B / 2 >= -84 for fM), so a
        // factor underflows only where the exact value does.
        {
            const int c = tid >> 1, par = tid & 1;     // channel; blocks 2 par and 2 par + 1
            const uint8_t *gcol = stg + ST_G + (c >> 6) * 8192 + ((c & 7) << 1);
            const int chk = (c & 63) >> 3;
            float Ls[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                float acc = 0.0f;
#pragma unroll
                for (int t = 0; t < 16; ++t)
                    acc += __bfloat162float(*(const __nv_bfloat16 *)(gcol + swz(16 * (2 * par + u) + t, chk)));
                Ls[u] = acc;
            }
            const float x0 = __shfl_xor_sync(0xffffffffu, Ls[0], 1), x1 = __shfl_xor_sync(0xffffffffu, Ls[1], 1);
            const float Lv[4] = {par ? x0 : Ls[0], par ? x1 : Ls[1], par ? Ls[0] : x0, par ? Ls[1] : x1};
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int Bq = 2 * par + u;
                float lpre = 0.0f, lpost = 0.0f;
#pragma unroll
                for (int J = 0; J < 4; ++J) {
                    if (J < Bq) lpre += Lv[J];
                    if (J > Bq) lpost += Lv[J];
                }
                const bool badB = !(Ls[u] >= BAD_LOG);
                const float fM = __expf((badB ? 0.0f : -0.5f * Ls[u]) - LN_SC);
                FT[FT_G + Bq * DD + c] = __expf(lpre);
                FT[FT_L + Bq * DD + c] = __expf(lpost);
                FT[FT_M + Bq * DD + c] = fM;
                FT[FT_D + Bq * DD + c] = badB ? 0.0f : fM;
                if (badB) atomicOr(&badmask[Bq * 4 + (c >> 5)], 1u << (c & 31));
#pragma unroll
                for (int I = 1; I < 4; ++I) {
                    if (I <= Bq) continue;
                    float l = Lv[I] >= BAD_LOG ? 0.5f * Lv[I] : 0.0f;
#pragma unroll
                    for (int J = 1; J < 3; ++J)
                        if (J > Bq && J < I) l += Lv[J];
                    FT[FT_C + fc_slot(Bq, I) * DD + c] = __expf(l);
                }
            }
            if (par == 0) GCsm[c] = __expf(Lv[0] + Lv[1] + Lv[2] + Lv[3]);
        }
        __syncthreads();
        // pass 2: per token.  Lane (qq, a) of warp (B, cb) takes tokens 16 B + 4 qq + s, s < 4,
        // and channels c0 .. c0 + 7.  With SC = 2^120:
        //   E1 = SC exp(G_i - G_blockstart)  (includes token i)
        //   E2 = SC exp(G_blockend - G_i)    (excludes token i)
        // from log-domain prefix sums, so no partial product can underflow; both are normal
        // numbers for block log-decays down to BAD_LOG (SC e^-168 ~ e^-84.8).
        {
            const int B = warp & 3;           // token block of this warp
            const int cb = warp >> 2;         // channel block (64 channels)
            const int qq = lane & 3;          // token quarter inside the block
            const int a = lane >> 2;          // 16-byte chunk (8 channels) inside the channel block
            const int c0 = 64 * cb + 8 * a;
            float Gin[4][8], Lb[8];
            {
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    const int i = 16 * B + 4 * qq + s;
                    float gf[8];
                    unpack8(*(const uint4 *)(stg + ST_G + cb * 8192 + swz(i, a)), gf);
#pragma unroll
                    for (int e = 0; e < 8; ++e) Gin[s][e] = (s == 0 ? 0.0f : Gin[s - 1][e]) + gf[e];
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    // exclusive prefix of the quarter log sums across the quad, and the block total
                    float l = Gin[3][e];
                    float y = __shfl_up_sync(0xffffffffu, l, 1, 4);
                    if (qq >= 1) l += y;
                    y = __shfl_up_sync(0xffffffffu, l, 2, 4);
                    if (qq >= 2) l += y;
                    y = __shfl_up_sync(0xffffffffu, l, 1, 4);
                    const float lex = qq >= 1 ? y : 0.0f;
                    Lb[e] = __shfl_sync(0xffffffffu, l, (lane & ~3) | 3);
#pragma unroll
                    for (int s = 0; s < 4; ++s) Gin[s][e] += lex;   // G_i - G_blockstart
                }
            }
            auto ftab = [&](int off, float (&f)[8]) {
                const float4 u0 = *(const float4 *)(FT + off + c0), u1 = *(const float4 *)(FT + off + c0 + 4);
                f[0] = u0.x; f[1] = u0.y; f[2] = u0.z; f[3] = u0.w; f[4] = u1.x; f[5] = u1.y; f[6] = u1.z; f[7] = u1.w;
            };
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                const int i = 16 * B + 4 * qq + s;
                const uint32_t off = cb * 8192 + swz(i, a);
                float qf[8], kf[8], o[8], E1[8], E2[8], f[8];
                unpack8(*(const uint4 *)(stg + ST_Q + off), qf);
                unpack8(*(const uint4 *)(stg + ST_K + off), kf);
                // exact diagonal of P: partial q_i . k_i over this lane's 8 channels
                float pd = 0.0f;
#pragma unroll
                for (int e = 0; e < 8; ++e) pd += qf[e] * kf[e];
                pd += __shfl_xor_sync(0xffffffffu, pd, 4);
                pd += __shfl_xor_sync(0xffffffffu, pd, 8);
                pd += __shfl_xor_sync(0xffffffffu, pd, 16);
                if (a == 0) PDsm[cb * CK + i] = pd;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    E1[e] = __expf(Gin[s][e] + LN_SC);
                    E2[e] = __expf(Lb[e] - Gin[s][e] + LN_SC);
                }
                // Q^ = Gamma q (fp32 K-major tile for the tf32 MMA), Gamma_i = (E1 / SC) fG;
                // odd quarters write their two 16-byte halves in the other order, which spreads
                // each store over all 32 banks
                ftab(FT_G + B * DD, f);
                float gam[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    gam[e] = (E1[e] * INV_SC) * f[e];
                    o[e] = qf[e] * gam[e];
                }
                {
                    uint8_t *qh = sm + OFF_QH + (2 * cb + (a >> 2)) * 8192;
                    const bool sw = qq & 1;
                    const float4 lo4 = make_float4(o[0], o[1], o[2], o[3]), hi4 = make_float4(o[4], o[5], o[6], o[7]);
                    *(float4 *)(qh + swz(i, 2 * (a & 3) + (sw ? 1 : 0))) = sw ? hi4 : lo4;
                    *(float4 *)(qh + swz(i, 2 * (a & 3) + (sw ? 0 : 1))) = sw ? lo4 : hi4;
                }
                // K^ = Gamma k (in place)
#pragma unroll
                for (int e = 0; e < 8; ++e) o[e] = kf[e] * gam[e];
                *(uint4 *)(stg + ST_K + off) = pack8(o);
                // K~ = exp(G_C - G_i) k (over g) = k (E2 / SC) fL
                ftab(FT_L + B * DD, f);
#pragma unroll
                for (int e = 0; e < 8; ++e) o[e] = kf[e] * ((E2[e] * INV_SC) * f[e]);
                *(uint4 *)(stg + ST_G + off) = pack8(o);
                // Gram rows [Q_B; K_B] scaled by E1 fM = exp(G_i - m_B): hi part to the Gram
                // rows, bf16 residual to X2 (free until the readback)
                ftab(FT_M + B * DD, f);
                const int rq = 32 * B + 4 * qq + s;
                {
                    float rf[8], hf[8], lo[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        rf[e] = E1[e] * f[e];
                        o[e] = qf[e] * rf[e];
                    }
                    const uint4 hq = pack8(o);
                    unpack8(hq, hf);
#pragma unroll
                    for (int e = 0; e < 8; ++e) lo[e] = o[e] - hf[e];
                    *(uint4 *)(gro + GR_R + cb * R_CB + swz(rq, a)) = hq;
                    *(uint4 *)(sm + OFF_X2 + cb * R_CB + swz(rq, a)) = pack8(lo);
#pragma unroll
                    for (int e = 0; e < 8; ++e) o[e] = kf[e] * rf[e];
                    const uint4 hk = pack8(o);
                    unpack8(hk, hf);
#pragma unroll
                    for (int e = 0; e < 8; ++e) lo[e] = o[e] - hf[e];
                    *(uint4 *)(gro + GR_R + cb * R_CB + swz(rq + 16, a)) = hk;
                    *(uint4 *)(sm + OFF_X2 + cb * R_CB + swz(rq + 16, a)) = pack8(lo);
                }
                // Gram columns, diagonal block: k E2 fD = k exp(m_B - G_j) (0 where L_B < BAD_LOG);
                // hi part to diagonal column row i, bf16 residual over the (now dead) raw q
                ftab(FT_D + B * DD, f);
                {
                    float hf[8], lo[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) o[e] = kf[e] * (E2[e] * f[e]);
                    const uint4 hc = pack8(o);
                    unpack8(hc, hf);
#pragma unroll
                    for (int e = 0; e < 8; ++e) lo[e] = o[e] - hf[e];
                    *(uint4 *)(gro + GR_CV + cb * CV_CB + swz(i, a)) = hc;
                    *(uint4 *)(stg + ST_Q + off) = pack8(lo);
                }
                // Gram columns for later blocks I > B: k (E2 / SC) fC(B, I)
#pragma unroll
                for (int I = 1; I < 4; ++I) {
                    if (I <= B) continue;
                    ftab(FT_C + fc_slot(B, I) * DD, f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) o[e] = kf[e] * ((E2[e] * INV_SC) * f[e]);
                    *(uint4 *)(gro + GR_CV + cb * CV_CB + swz(cv_off(I) + i, a)) = pack8(o);
                }
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();

        // ============================================================ Gram + O init (MMA), decay S
        if (tid == 0) {
            tc_fence_after();
            const uint32_t sR = smem_u32(gro + GR_R), sCV = smem_u32(gro + GR_CV);
            for (int kk = 0; kk < 8; ++kk)
                mma_ss(tmem + TM_G, sdesc(sR + (kk >> 2) * R_CB + (kk & 3) * 32, 16, 1024),
                       sdesc(sCV + (kk >> 2) * CV_CB + (kk & 3) * 32, 16, 1024), id_gram, kk > 0);
            // diagonal-block residual: R_lo x CVd (CV rows 0..63) + R x CVd_lo (over the q tile)
            const uint32_t sRL = smem_u32(sm + OFF_X2), sCVL = smem_u32(stg + ST_Q);
            for (int kk = 0; kk < 8; ++kk)
                mma_ss(tmem + TM_CORR, sdesc(sRL + (kk >> 2) * R_CB + (kk & 3) * 32, 16, 1024),
                       sdesc(sCV + (kk >> 2) * CV_CB + (kk & 3) * 32, 16, 1024), id_corr, kk > 0);
            for (int kk = 0; kk < 8; ++kk)
                mma_ss(tmem + TM_CORR, sdesc(sR + (kk >> 2) * R_CB + (kk & 3) * 32, 16, 1024),
                       sdesc(sCVL + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024), id_corr, 1);
            // O^T = S^T Q^^T at tf32: A = fp32 state in TMEM, 8 key channels per MMA
            const uint32_t sQ = smem_u32(sm + OFF_QH);
            for (int kk = 0; kk < 16; ++kk)
                mma_ts_tf32(tmem + TM_O, tmem + TM_S + kk * 8, sdesc(sQ + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024),
                            id_o0, kk > 0);
            mma_commit(bar_mma);
        }
        if (!mma_wait()) break;
        tc_fence_after();
        if (tid == 0 && n + 1 < nchunks) issue_tma(n + 1);   // the Gram region is free now

        // ============================================================ Gram readback -> P, A
        {
            const int I = warp & 3;
            const bool is_q = lane < 16;
            const int i = 16 * I + (lane & 15);
            const int ncol = 8 * (I + 1);                 // this warp's share of CV_I
            const int jbase = half * ncol;
            const float bi = BETAsm[i];
            const float pdiag = PDsm[i] + PDsm[CK + i];   // exact q_i . k_i
            const uint32_t *bmask = badmask + 4 * I;
            // the warp's TMEM loads go out in two batches (earlier-block columns, then the
            // diagonal block with its residual), one wait each; chunks are counted from the
            // warp's last 8 columns, so only mm = 0, 1 can be diagonal
            auto emit = [&](int j0, const uint32_t (&r)[8]) {
                float vals[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int j = j0 + e;
                    const float v = __uint_as_float(r[e]);
                    if (is_q) vals[e] = j < i ? v : (j == i ? pdiag : 0.0f);
                    else vals[e] = j < i ? bi * v : 0.0f;
                }
                if (is_q) {
                    float lo[8];
                    const uint4 hi = pack8(vals);
                    float hf[8];
                    unpack8(hi, hf);
#pragma unroll
                    for (int e = 0; e < 8; ++e) lo[e] = vals[e] - hf[e];
                    *(uint4 *)(sm + OFF_P + swz(i, j0 >> 3)) = hi;
                    *(uint4 *)(sm + OFF_PL + swz(i, j0 >> 3)) = pack8(lo);
                } else {
                    *(float4 *)(A32 + i * 64 + j0) = make_float4(vals[0], vals[1], vals[2], vals[3]);
                    *(float4 *)(A32 + i * 64 + j0 + 4) = make_float4(vals[4], vals[5], vals[6], vals[7]);
                }
            };
            {
                uint32_t r[4][8];
#pragma unroll
                for (int mm = 0; mm < 4; ++mm) {
                    const int j0 = jbase + 8 * (I - mm);
                    if (mm <= I && j0 < 16 * I) tmem_ld8(tmem + lane_q + TM_G + cv_off(I) + j0, r[mm]);
                }
                tmem_wait_ld();
#pragma unroll
                for (int mm = 0; mm < 4; ++mm) {
                    const int j0 = jbase + 8 * (I - mm);
                    if (mm <= I && j0 < 16 * I) emit(j0, r[mm]);
                }
            }
            {
                uint32_t r[2][8], c8[2][8];
#pragma unroll
                for (int mm = 0; mm < 2; ++mm) {
                    const int j0 = jbase + 8 * (I - mm);
                    if (mm <= I && j0 >= 16 * I) {
                        tmem_ld8(tmem + lane_q + TM_G + j0, r[mm]);
                        tmem_ld8(tmem + lane_q + TM_CORR + j0, c8[mm]);
                    }
                }
                tmem_wait_ld();
#pragma unroll
                for (int mm = 0; mm < 2; ++mm) {
                    const int j0 = jbase + 8 * (I - mm);
                    if (mm <= I && j0 >= 16 * I) {
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            r[mm][e] = __float_as_uint(__uint_as_float(r[mm][e]) + __uint_as_float(c8[mm][e]));
                        emit(j0, r[mm]);
                    }
                }
            }
            // exact diagonal-block terms of channels whose block decay underflows the Gram
            // factorisation, added in place to this thread's own entries (rare path)
            for (int wd = 0; wd < 4; ++wd) {
                for (uint32_t m = bmask[wd]; m != 0u; m &= m - 1u) {
                    const int c = 32 * wd + __ffs((int)m) - 1;
                    const size_t rowi = ((size_t)(b * T + t0 + i) * p.H + h) * DD + c;
                    const float xi = (t0 + i < T) ? __bfloat162float((is_q ? p.q : p.k)[rowi]) : 0.0f;
                    float w = 1.0f;   // exp(G_i - G_j), built backwards from j = i
                    for (int j = i; j >= 16 * I; --j) {
                        const bool valid = t0 + j < T;
                        const size_t rowj = ((size_t)(b * T + t0 + j) * p.H + h) * DD + c;
                        if (j < i && j >= jbase && j < jbase + ncol) {
                            const float d = xi * (valid ? __bfloat162float(p.k[rowj]) : 0.0f) * w;
                            if (is_q) {
                                __nv_bfloat16 *ph = (__nv_bfloat16 *)(sm + OFF_P + swz(i, j >> 3)) + (j & 7);
                                __nv_bfloat16 *pl = (__nv_bfloat16 *)(sm + OFF_PL + swz(i, j >> 3)) + (j & 7);
                                const float v = __bfloat162float(*ph) + __bfloat162float(*pl) + d;
                                const __nv_bfloat16 vh = __float2bfloat16_rn(v);
                                *ph = vh;
                                *pl = __float2bfloat16_rn(v - __bfloat162float(vh));
                            } else {
                                A32[i * 64 + j] += bi * d;
                            }
                        }
                        w *= __expf(valid ? __bfloat162float(p.g[rowj]) : 0.0f);
                    }
                }
            }
            if (half == 1) {
                for (int jc = 2 * (I + 1); jc < 8; ++jc) {
                    if (is_q) {
                        *(uint4 *)(sm + OFF_P + swz(i, jc)) = make_uint4(0, 0, 0, 0);
                        *(uint4 *)(sm + OFF_PL + swz(i, jc)) = make_uint4(0, 0, 0, 0);
                    } else {
                        *(float4 *)(A32 + i * 64 + 8 * jc) = make_float4(0.f, 0.f, 0.f, 0.f);
                        *(float4 *)(A32 + i * 64 + 8 * jc + 4) = make_float4(0.f, 0.f, 0.f, 0.f);
                    }
                }
            }
        }
        __syncthreads();
        if (tid < 16) badmask[tid] = 0u;   // masks consumed

        // ============================================================ T = (I + A)^{-1} Diag(beta)
        // L = I + A, blocked by 16: diagonal inverses L_II^{-1} (right-looking forward
        // substitution, one column per thread), then A''_IK = L_II^{-1} A_IK, then block rows
        // by distance: T_IJ = -sum_{K=J}^{I-1} A''_IK T_KJ.  The block products run on
        // strips of 4 rows x 1 column per thread (row segments read as float4).
        if (tid < 64) {
            const int Ib = tid >> 4, col = tid & 15;
            const float *Ab = A32 + (16 * Ib) * 64 + 16 * Ib;
            float x[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) x[r] = r == col ? 1.0f : 0.0f;
#pragma unroll
            for (int m = 0; m < 15; ++m)
#pragma unroll
                for (int r = m + 1; r < 16; ++r) x[r] -= Ab[r * 64 + m] * x[m];
#pragma unroll
            for (int r = 0; r < 16; ++r) LINV[(16 * Ib + r) * 64 + 16 * Ib + col] = x[r];
        }
        __syncthreads();
        {
            const int set = tid >> 6;               // which block product this thread serves
            const int r0 = ((tid >> 4) & 3) * 4;    // rows r0..r0+3 of the 16x16 block
            const int cc = tid & 15;                // column
            // acc[q] += sum_m X[rowbase + r0 + q][colX + m] * Y[rowY + m][colY + cc]
            auto strip = [&](const float *X, int xrow, int xcol, const float *Y, int yrow, int ycol,
                             float (&acc)[4]) {
#pragma unroll
                for (int m4 = 0; m4 < 16; m4 += 4) {
                    const float y0 = Y[(yrow + m4 + 0) * 64 + ycol + cc], y1 = Y[(yrow + m4 + 1) * 64 + ycol + cc];
                    const float y2 = Y[(yrow + m4 + 2) * 64 + ycol + cc], y3 = Y[(yrow + m4 + 3) * 64 + ycol + cc];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float4 xv = *(const float4 *)(X + (xrow + r0 + q) * 64 + xcol + m4);
                        acc[q] += xv.x * y0 + xv.y * y1 + xv.z * y2 + xv.w * y3;
                    }
                }
            };
            // A''_IK for the 6 pairs (I, K), K < I: sets 0..3 take pairs {set, set + 4}
            float y[2][4];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int pi = set + 4 * u;
#pragma unroll
                for (int q = 0; q < 4; ++q) y[u][q] = 0.0f;
                if (pi < 6) {
                    const int I = pi < 1 ? 1 : (pi < 3 ? 2 : 3);
                    const int K = pi < 1 ? 0 : (pi < 3 ? pi - 1 : pi - 3);
                    strip(LINV, 16 * I, 16 * I, A32, 16 * I, 16 * K, y[u]);
                }
            }
            __syncthreads();
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int pi = set + 4 * u;
                if (pi < 6) {
                    const int I = pi < 1 ? 1 : (pi < 3 ? 2 : 3);
                    const int K = pi < 1 ? 0 : (pi < 3 ? pi - 1 : pi - 3);
#pragma unroll
                    for (int q = 0; q < 4; ++q) A32[(16 * I + r0 + q) * 64 + 16 * K + cc] = y[u][q];
                }
            }
            __syncthreads();
#pragma unroll
            for (int d = 1; d < 4; ++d) {
                const int J = set, I = set + d;
                if (I < 4) {
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int K = 0; K < 3; ++K)
                        if (K >= J && K < I) strip(A32, 16 * I, 16 * K, LINV, 16 * K, 16 * J, acc);
#pragma unroll
                    for (int q = 0; q < 4; ++q) LINV[(16 * I + r0 + q) * 64 + 16 * J + cc] = -acc[q];
                }
                __syncthreads();
            }
        }
        for (int idx = tid; idx < 64 * 8; idx += NT) {
            const int i = idx >> 3, jc = idx & 7;
            float vals[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int j = 8 * jc + e;
                vals[e] = j <= i ? LINV[i * 64 + j] * BETAsm[j] : 0.0f;
            }
            *(uint4 *)(sm + OFF_T + swz(i, jc)) = pack8(vals);
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();

        // ============================================================ W^T = K^^T T^T, U~^T = V^T T^T
        if (tid == 0) {
            tc_fence_after();
            const uint32_t sK = smem_u32(stg + ST_K), sV = smem_u32(stg + ST_V), sT_ = smem_u32(sm + OFF_T);
            for (int kk = 0; kk < 4; ++kk)
                mma_ss(tmem + TM_W, sdesc(sK + kk * 2048, 8192, 1024), sdesc(sT_ + kk * 32, 16, 1024), id_wt, kk > 0);
            for (int kk = 0; kk < 4; ++kk)
                mma_ss(tmem + TM_U, sdesc(sV + kk * 2048, 8192, 1024), sdesc(sT_ + kk * 32, 16, 1024), id_wt, kk > 0);
            mma_commit(bar_mma);
        }
        if (!mma_wait()) break;
        tc_fence_after();
        {
            // W^T (lane = key channel c = 32 (warp & 3) + lane) -> W in shared memory, fp32 K-major [i][c]
            uint32_t r[32];
            tmem_ld32(tmem + lane_q + TM_W + 32 * half, r);
            tmem_wait_ld();
            // K-block c / 32 = this warp's lane quarter; a warp writes one 128-byte row per token i
            uint8_t *wb = sm + OFF_W + (warp & 3) * 8192 + (lane & 3) * 4;
#pragma unroll
            for (int e = 0; e < 32; ++e)
                *(uint32_t *)(wb + swz(32 * half + e, lane >> 2)) = r[e];
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            // U^T -= S^T W^T at tf32: A = fp32 state in TMEM, B = W fp32 K-major
            const uint32_t sW = smem_u32(sm + OFF_W);
            for (int kk = 0; kk < 16; ++kk)
                mma_ts_tf32(tmem + TM_U, tmem + TM_S + kk * 8, sdesc(sW + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024),
                            id_u, 1);
            mma_commit(bar_mma);
        }
        if (!mma_wait()) break;
        tc_fence_after();
        {
            // U^T fp32 -> bf16 hi and lo A operands
            uint32_t r[32], r8[8], l8[8];
            tmem_ld32(tmem + lane_q + TM_U + 32 * half, r);
            tmem_wait_ld();
#pragma unroll
            for (int m = 0; m < 2; ++m) {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float x0 = __uint_as_float(r[16 * m + 2 * e]), x1 = __uint_as_float(r[16 * m + 2 * e + 1]);
                    r8[e] = pack_bf16x2(x0, x1);
                    const float2 hv = unpack_bf16x2(r8[e]);
                    l8[e] = pack_bf16x2(x0 - hv.x, x1 - hv.y);
                }
                tmem_st8(tmem + lane_q + TM_UB + 16 * half + 8 * m, r8);
                tmem_st8(tmem + lane_q + TM_UL + 16 * half + 8 * m, l8);
            }
            // S^T <- S^T Diag(exp G_C) (every reader of the chunk-start state has finished)
            for (int cc = 0; cc < 64; cc += 32) {
                const uint32_t ta = tmem + lane_q + TM_S + 64 * half + cc;
                tmem_ld32(ta, r);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    r[e] = __float_as_uint(__uint_as_float(r[e]) * GCsm[64 * half + cc + e]);
                tmem_st32(ta, r);
            }
            tmem_wait_st();
        }
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint32_t sP = smem_u32(sm + OFF_P), sPL = smem_u32(sm + OFF_PL), sG = smem_u32(stg + ST_G);
            for (int kk = 0; kk < 4; ++kk) {
                mma_ts(tmem + TM_O, tmem + TM_UB + kk * 8, sdesc(sP + kk * 32, 16, 1024), id_op, 1);
                mma_ts(tmem + TM_O, tmem + TM_UL + kk * 8, sdesc(sP + kk * 32, 16, 1024), id_op, 1);
                mma_ts(tmem + TM_O, tmem + TM_UB + kk * 8, sdesc(sPL + kk * 32, 16, 1024), id_op, 1);
            }
            for (int kk = 0; kk < 4; ++kk) {
                mma_ts(tmem + TM_S, tmem + TM_UB + kk * 8, sdesc(sG + kk * 2048, 8192, 1024), id_s, 1);
                mma_ts(tmem + TM_S, tmem + TM_UL + kk * 8, sdesc(sG + kk * 2048, 8192, 1024), id_s, 1);
            }
            mma_commit(bar_mma);
        }
        if (!mma_wait()) break;
        tc_fence_after();
        {
            // O^T -> bf16 tile in X2 (the load tiles' layout: 2 channel blocks of [64 rows x 128 B],
            // 128-byte swizzle), then two TMA stores; rows past T are clipped by the tensor map
            const int v = 32 * (warp & 3) + lane;
            uint32_t r[32];
            tmem_ld32(tmem + lane_q + TM_O + 32 * half, r);
            tmem_wait_ld();
            uint8_t *ot = sm + OFF_X2 + (v >> 6) * 8192 + ((v & 7) << 1);
#pragma unroll
            for (int e = 0; e < 32; ++e)
                *(__nv_bfloat16 *)(ot + swz(32 * half + e, (v & 63) >> 3)) = __float2bfloat16_rn(__uint_as_float(r[e]));
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tma_store_4d(&tm_o, sm + OFF_X2, 0, h, t0, b);
            tma_store_4d(&tm_o, sm + OFF_X2 + 8192, 64, h, t0, b);
            bulk_commit();
        }
    }

    // ---------------------------------------------------------------- final state
    if (p.sT && !*abort_flag) {
        tc_fence_after();
        const int v = 32 * (warp & 3) + lane;
        float *sT = p.sT + (size_t)bh * DD * DD;
        for (int cc = 0; cc < 64; cc += 32) {
            uint32_t r[32];
            tmem_ld32(tmem + lane_q + TM_S + 64 * half + cc, r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) sT[(size_t)(64 * half + cc + e) * DD + v] = __uint_as_float(r[e]);
        }
    }
    if (tid == 0) bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)f;
        else
            cudaGetLastError();
    });
    return fn;
}

// [B, T, H, 128] bf16 -> 4-D map (128, H, T, B), box (64, 1, 64, 1), 128-byte swizzle,
// zero fill past T.
bool make_map(CUtensorMap *m, const void *base, int B, int T, int H)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)DD, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)DD * 2, (cuuint64_t)H * DD * 2, (cuuint64_t)T * H * DD * 2};
    cuuint32_t box[4] = {64, 1, 64, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool device_is_sm100()
{
    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return false;
    return major == 10 && minor == 0;
}

}  // namespace

bool chunk_tc_supported(const ChunkArgs &a)
{
    return a.io == IO_BF16 && a.dk == DD && a.dv == DD && !a.qkv_f32 && !a.g_f32 && !a.beta_f32 && !a.out_f32 &&
           a.T > 0 && device_is_sm100() && encode_fn() != nullptr;
}

cudaError_t launch_chunk_tc(const ChunkArgs &a, cudaStream_t s)
{
    CUtensorMap mq, mk, mv, mg, mo;
    if (!make_map(&mq, a.q, a.B, a.T, a.H) || !make_map(&mk, a.k, a.B, a.T, a.H) ||
        !make_map(&mv, a.v, a.B, a.T, a.H) || !make_map(&mg, a.g, a.B, a.T, a.H) ||
        !make_map(&mo, a.out, a.B, a.T, a.H))
        return cudaErrorInvalidValue;
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(kda_chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    });
    if (attr_err != cudaSuccess) return attr_err;
    TcParams p{(const __nv_bfloat16 *)a.q, (const __nv_bfloat16 *)a.k, (const __nv_bfloat16 *)a.g,
               (const __nv_bfloat16 *)a.beta, a.s0, (__nv_bfloat16 *)a.out, a.sT, a.T, a.H, a.err};
    kda_chunk_tc_kernel<<<a.B * a.H, NT, SMEM_BYTES, s>>>(mq, mk, mv, mg, mo, p);
    return cudaGetLastError();
}

}  // namespace kda
