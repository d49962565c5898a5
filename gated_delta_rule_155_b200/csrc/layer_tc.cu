// layer_tc.cu — the KDA layer core in one tcgen05 kernel (bf16 I/O, dk = dv = 128).
//
// Per (b, h) head, chunks of C = 32 tokens in order, fp32 state in tensor memory (transposed:
// lane = value column v, column = key channel c).  Per chunk:
//
//   pass A (CUDA cores)  prologue from the raw bf16 tiles: causal depthwise conv of kernel 4
//                        (PyTorch Conv1d tap order, history from the previous chunk's tiles,
//                        zero before the sequence) + SiLU for q, k, v; the partial sums of
//                        squares of the q and k rows; g = max(-exp(A_log) softplus(g_raw +
//                        dt_bias), bound) and its in-half prefix; beta = sigmoid(b_raw)
//                        (open-model-atlas "Kimi-K3" linear_attn_config: short_conv_kernel_size
//                        4, gate_lower_bound; maxtext PR #5548 review item 2: exp(A_log) drives
//                        the decay, conv weights and dt_bias in F32)
//   pass B               per-(block, channel) decay factors (blocks of 16 tokens)
//   pass C               q, k L2-normalised; Q^ = Gamma q, K^ = Gamma k, K~ = exp(G_C - G) k,
//                        V, and the Gram operands (the overflow-safe midpoint factorisation of
//                        the tensor-core prefill, chunk_tc.cu)
//   Gram (tcgen05)       P (j <= i) and A (j < i): R_hi [CV_hi; CV_lo] (M = 128, N = 96) and
//                        R_lo CV_hi (N = 48), K = 128
//   inverse || Y, O init T = (I + A)^{-1} Diag(beta), one column per lane in registers, while
//                        the tensor cores compute Y^T = S^T K^^T and O^T = S^T Q^^T
//   U, O, S (tcgen05)    U = T (V - Y);  O += P U;  S <- Diag(exp G_C) S + K~^T U
//   epilogue             out = gain * cast_bf16(o * rsqrt(mean_v(o^2) + eps)) * sigmoid(z)
//                        (atlas.klimoza.dev "Kimi-K3 > KDA layers", KimiRMSNorm excerpt;
//                         maxtext PR #5543: sigmoid output gate), staged and stored by TMA
//
// Precision.  The RMSNorm rescales each output row to unit RMS, so a row whose o is small
// next to the terms that make it up amplifies every rounding of the chunk algebra (a single
// bf16 rounding of q or k puts such rows at many times the tolerance).  Every operand of
// every MMA therefore enters as a bf16 hi + lo pair (three products: a_hi b_hi + a_lo b_hi +
// a_hi b_lo, about 2^-16 relative): the Gram rows and columns, T, V, Y, U, P, K~, Q^ and the
// state; K^ (in Y = K^ S) alone is one bf16 rounding.  The diagonal of P is the exact q_i.k_i.
// With 32-token chunks all those pairs and a double-buffered stage fit in shared memory
// (about 210 KB); the prefill kernel's 64-token chunks keep fewer of them.
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace kda {
namespace {

using namespace tc;

constexpr int NT = 512;       // 16 warps
constexpr int CK = 32;        // chunk
constexpr int DD = 128;       // dk = dv
constexpr float BAD_LOG = -168.0f;   // block log-decays below this take the exact diagonal path
constexpr float L2_EPS = 1e-6f;

// ---------------------------------------------------------------- shared memory (1024-aligned base)
// A tile is [32 rows][128 channels] bf16 as two 64-channel blocks of [32 rows][128 B] with the
// 128-byte swizzle (the TMA box layout); element (i, c) at (c >> 6) * CBT + swz(i, (c & 63) >> 3).
constexpr int CBT = 4096, TILE = 2 * CBT;
// stage (one per chunk parity): raw q, k, v, g and the output gate z; the g tile (dead after
// pass A) stages the chunk's output for its TMA store
constexpr int ST_Q = 0, ST_K = TILE, ST_V = 2 * TILE, ST_G = 3 * TILE, ST_Z = 4 * TILE;
constexpr int STAGE = 5 * TILE;
constexpr int OFF_STG0 = 0, OFF_STG1 = STAGE;
// Gram region: rows R = [Q_0; K_0; Q_1; K_1] (64 rows x 128 channels, hi and lo, K-major), the
// M = 128 MMA also reads the 64 rows after each channel block (other operands; the tensor-memory
// lanes they produce are never read); columns CV (48 rows: tokens 0..31 with their own block's
// reference, then block 0's tokens with block 1's), hi then lo in one 96-row block per channel
// block, so that R_hi [CV_hi; CV_lo] is one N = 96 MMA.  After the Gram: P hi, lo and T
// hi, lo ([32 rows][128 B], K-major, columns 0..31 used) and A (fp32 [32][AST], row-major).
constexpr int OFF_GR = 2 * STAGE;
constexpr int R_CB = 8192, CV_CB = 12288, CV_LO = 6144;   // CV_lo rows follow CV_hi in a block
constexpr int GR_RH = 0, GR_RL = 16384, GR_CV = 32768;
constexpr int GR_BYTES = GR_CV + 2 * CV_CB;
constexpr int GR_PH = 0, GR_PL = 4096, GR_TH = 8192, GR_TL = 12288, GR_A = 16384, AST = 36;
// operand tiles ([32 rows][128 channels] bf16, the tile layout)
// [Q^_hi; K^] per channel block (32 + 32 rows): one N = 64 B operand gives O and Y into adjacent
// tensor-memory columns; then Q^ lo (the tile layout)
constexpr int OFF_QK = OFF_GR + GR_BYTES, QK_CB = 8192, QK_K = 4096;
constexpr int OFF_QL = OFF_QK + 2 * QK_CB;
constexpr int OFF_KTH = OFF_QL + TILE, OFF_KTL = OFF_KTH + TILE;    // K~ hi, lo (MN-major B of the state update)
constexpr int OFF_VH = OFF_KTL + TILE, OFF_VL = OFF_VH + TILE;      // V hi, lo (MN-major A of U)
constexpr int OFF_CW = OFF_VL + TILE;                               // conv weights fp32 [3][128][4]
// per-(block, channel) table, fp32 rows of FSTRIDE: fG, fL, fM for blocks 0, 1; the half-block
// log-decays (row FT_HS + 2 B + half); fC, block 1's reference for block 0's columns
constexpr int FSTRIDE = 136;
constexpr int FT_G = 0, FT_L = 2, FT_M = 4, FT_HS = 6, FT_C = 10, FT_ROWS = 11;
constexpr int OFF_FT = OFF_CW + 3 * DD * 4 * 4;
constexpr int OFF_MISC = OFF_FT + FT_ROWS * FSTRIDE * 4;
constexpr int MS_BADMASK = 0;      // uint32 [2][4]: channels whose block log-decay is below BAD_LOG
constexpr int MS_GC = 32;          // fp32 [128] exp(G_C)
constexpr int MS_BETA = 544;       // fp32 [32]
constexpr int MS_PD = 672;         // fp32 [4][32] exact q_i . k_i per channel quarter
constexpr int MS_NRM = 1184;       // fp32 [2][4][32] sums of squares of the conv outputs of q, k
constexpr int MS_RMS = 2208;       // fp32 [4][32] sums of o^2 per lane quarter
constexpr int MS_BRAW = 2720;      // uint32 [2][32] b_raw words in flight (cp.async)
constexpr int MS_DTB = 2976;       // fp32 [128] dt_bias
constexpr int MS_GAIN = 3488;      // fp32 [128] RMSNorm gain
constexpr int MS_BAR = 4000;       // uint64: tma0, tma1, mma, y, o init, o, drain
constexpr int MS_TSLOT = 4064, MS_ABORT = 4068;
constexpr int MISC_BYTES = 4096;
constexpr int SMEM_BYTES = OFF_MISC + MISC_BYTES + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory per block");
static_assert(OFF_GR % 1024 == 0 && OFF_QK % 1024 == 0 && OFF_VL % 1024 == 0 && GR_CV % 1024 == 0 &&
              CV_LO % 1024 == 0, "operand tiles are 1024-aligned");
static_assert(GR_A + 32 * AST * 4 <= GR_BYTES && OFF_MISC % 16 == 0, "layout");

// tensor memory columns
constexpr uint32_t TM_S = 0;     // fp32 S^T, 128
constexpr uint32_t TM_SH = 128;  // bf16 S^T hi (two per column), 64
constexpr uint32_t TM_SL = 192;  // bf16 S^T lo, 64
constexpr uint32_t TM_G = 256;   // Gram D (lanes 0..63): R CV_hi in 48 columns, R_hi CV_lo in the next 48
constexpr uint32_t TM_O = 304;   // O^T, 32 (after the Gram readback)
constexpr uint32_t TM_Y = 336;   // Y^T, 32 (right after O: one N = 64 accumulator)
constexpr uint32_t TM_U = 368;   // U^T, 32
constexpr uint32_t TM_HI = 400;  // bf16 Y^T hi, then U^T hi, 16
constexpr uint32_t TM_LO = 416;  // bf16 Y^T lo, then U^T lo, 16

struct LayerTcParams {
    const __nv_bfloat16 *q, *k, *g, *b;   // raw q, k, gate input; b_raw [tokens, H]
    const float *conv_q, *conv_k, *conv_v, *A_log, *dt_bias, *gain;
    float g_lb, eps;
    const float *s0;
    float *sT;
    __nv_bfloat16 *out;
    int T, H;
    int *err;
    const int *cu;                 // packed sequence offsets, or null
    unsigned long long wait_ns;
    int skip_load_chunk;
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
// Activations with the fast reciprocal and logarithm (relative errors about 2^-21, well below
// the 2^-16 the chunk algebra keeps): the IEEE division and log1pf cost several times more.
KDA_DEVICE float silu_fast(float x) { return __fdividef(x, 1.0f + __expf(-x)); }
KDA_DEVICE float sigmoid_fast(float x) { return __fdividef(1.0f, 1.0f + __expf(-x)); }
// log(1 + e^x) = max(x, 0) + log(1 + e^-|x|); 1 + e^-|x| lies in (1, 2], where the logarithm
// keeps its relative accuracy
KDA_DEVICE float softplus_fast(float x) { return fmaxf(x, 0.0f) + __logf(1.0f + __expf(-fabsf(x))); }

// x -> bf16 hi and the bf16 residual lo
KDA_DEVICE void split8(const float (&x)[8], uint4 &hi, uint4 &lo)
{
    float hf[8], r[8];
    hi = pack8(x);
    unpack8(hi, hf);
#pragma unroll
    for (int e = 0; e < 8; ++e) r[e] = x[e] - hf[e];
    lo = pack8(r);
}

template <bool PACKED>
__global__ void __launch_bounds__(NT, 1)
kda_layer_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                    const __grid_constant__ CUtensorMap tm_z, const __grid_constant__ CUtensorMap tm_o,
                    LayerTcParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *misc = sm + OFF_MISC;
    uint8_t *gr = sm + OFF_GR;
    uint32_t *badmask = (uint32_t *)(misc + MS_BADMASK);
    float *FT = (float *)(sm + OFF_FT);
    float *CW = (float *)(sm + OFF_CW);
    float *GCsm = (float *)(misc + MS_GC);
    float *BETAsm = (float *)(misc + MS_BETA);
    float *PDsm = (float *)(misc + MS_PD);
    float *NRM = (float *)(misc + MS_NRM);
    float *RMS = (float *)(misc + MS_RMS);
    uint32_t *BRAW = (uint32_t *)(misc + MS_BRAW);
    float *DTB = (float *)(misc + MS_DTB);
    float *GAIN = (float *)(misc + MS_GAIN);
    uint64_t *bar_tma = (uint64_t *)(misc + MS_BAR);
    uint64_t *bar_mma = bar_tma + 2;
    uint64_t *bar_y = bar_tma + 3;
    uint64_t *bar_oi = bar_tma + 4;
    uint64_t *bar_o = bar_tma + 5;
    uint64_t *bar_drain = bar_tma + 6;
    uint32_t *tslot = (uint32_t *)(misc + MS_TSLOT);
    volatile int *abort_flag = (volatile int *)(misc + MS_ABORT);
    float *A32 = (float *)(gr + GR_A);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x, b = bh / p.H, h = bh % p.H;
    const SeqSpan span = PACKED ? seq_span(p.cu, b, p.T) : SeqSpan{b * p.T, p.T};
    const int T = span.len, row0 = span.row0;
    const int tt0 = PACKED ? row0 : 0, tb = PACKED ? 0 : b;
    const int nchunks = (T + CK - 1) / CK;
    const int lq = warp & 3, cg = warp >> 2;
    const uint32_t lane_q = (uint32_t)(32 * lq) << 16;

    if (tid == 0) {
        for (int x = 0; x < 7; ++x) mbar_init(&bar_tma[x], 1);
        mbar_init(bar_drain, 2);   // the two MMA-issuing threads
        *abort_flag = 0;
        for (int x = 0; x < 8; ++x) badmask[x] = 0u;
        fence_mbar_init();
        prefetch_tmap(&tm_q); prefetch_tmap(&tm_k); prefetch_tmap(&tm_v); prefetch_tmap(&tm_g);
        prefetch_tmap(&tm_z); prefetch_tmap(&tm_o);
    }
    if (warp == 0) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    // per-head constants: conv taps [tensor][channel][4], dt_bias, gain
    for (int x = tid; x < 3 * DD; x += NT) {
        const float *w = x < DD ? p.conv_q : (x < 2 * DD ? p.conv_k : p.conv_v);
        *(float4 *)(CW + 4 * x) = *(const float4 *)(w + ((size_t)h * DD + (x & (DD - 1))) * 4);
    }
    if (tid < DD) {
        DTB[tid] = p.dt_bias ? p.dt_bias[(size_t)h * DD + tid] : 0.0f;
        GAIN[tid] = p.gain ? p.gain[tid] : 1.0f;
    }
    const float gscale = __expf(p.A_log[h]);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;

    int tma_issued = 0, tma_consumed = 0;
    auto issue_tma = [&](int n) {
        if (n == p.skip_load_chunk) return;   // injected failure: the wait for it runs out
        ++tma_issued;
        const int r = n & 1;
        uint8_t *st = sm + (r ? OFF_STG1 : OFF_STG0);
        const int t0 = tt0 + n * CK;
        mbar_arrive_expect_tx(&bar_tma[r], 5 * TILE);
        for (int cb = 0; cb < 2; ++cb) {
            tma_load_4d(st + ST_Q + cb * CBT, &tm_q, cb * 64, h, t0, tb, &bar_tma[r]);
            tma_load_4d(st + ST_K + cb * CBT, &tm_k, cb * 64, h, t0, tb, &bar_tma[r]);
            tma_load_4d(st + ST_V + cb * CBT, &tm_v, cb * 64, h, t0, tb, &bar_tma[r]);
            tma_load_4d(st + ST_G + cb * CBT, &tm_g, cb * 64, h, t0, tb, &bar_tma[r]);
            tma_load_4d(st + ST_Z + cb * CBT, &tm_z, cb * 64, h, t0, tb, &bar_tma[r]);
        }
    };
    if (tid == 0 && nchunks > 0) issue_tma(0);

    {
        // initial state: S^T, lane v = value column, column c = key channel
        const int v = 32 * lq + lane;
        const float *s0 = p.s0 ? p.s0 + (size_t)bh * DD * DD : nullptr;
        uint32_t r[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(s0 ? s0[(size_t)(32 * cg + e) * DD + v] : 0.0f);
        tmem_st32(tmem + lane_q + TM_S + 32 * cg, r);
        tmem_wait_st();
    }

    uint32_t mma_phase = 0;
    // A wait that gives up sets *abort_flag; the flag is read only right after a block barrier
    // and before any TMA or MMA issue, so the whole CTA leaves the chunk loop at the same point.
    auto mma_wait = [&]() {
        mbar_wait_bounded(bar_mma, mma_phase, abort_flag, p.err, p.wait_ns);
        mma_phase ^= 1u;
    };

    constexpr uint32_t id_gram = idesc_bf16(128, 48, false, false);
    constexpr uint32_t id_gram96 = idesc_bf16(128, 96, false, false);
    constexpr uint32_t id_n64 = idesc_bf16(128, 64, false, false);
    static_assert(TM_Y == TM_O + 32 && TM_G + 96 <= TM_HI, "accumulator layout");
    constexpr uint32_t id_n32 = idesc_bf16(128, 32, false, false);
    constexpr uint32_t id_n32_neg = idesc_bf16(128, 32, false, false, true);
    constexpr uint32_t id_v = idesc_bf16(128, 32, true, false);
    constexpr uint32_t id_s = idesc_bf16(128, 128, false, true);

    // b_raw of the next chunk, global -> shared one chunk ahead (the aligned word that holds it)
    auto b_async = [&](int nn) {   // tid < CK
        const int t = nn * CK + tid;
        const void *src = p.b;
        uint32_t bytes = 0;
        if (t < T) {
            const uintptr_t ea = (uintptr_t)(p.b + (size_t)(row0 + t) * p.H + h);
            bytes = (ea & 2) ? 4u : 2u;
            src = (const void *)(ea & ~(uintptr_t)3);
        }
        cp_async4(smem_u32(BRAW + (nn & 1) * CK + tid), src, bytes);
        cp_async_commit();
    };
    if (tid < CK && nchunks > 0) b_async(0);

    constexpr float INV_SC = 7.523164e-37f;    // SC = 2^120
    constexpr float LN_SC = 83.17766f;         // 120 ln 2
    // Token mapping of passes A and C: warp (Bk, cq, th), lane (pp, a4): token i = 16 Bk + 8 th +
    // pp, channels c0 .. c0 + 7 with c0 = 32 cq + 8 a4 (16-byte chunk a of channel block cb).
    const int Bk = warp & 1, cq = (warp >> 1) & 3, th = warp >> 3;
    const int pp = lane & 7, a4 = lane >> 3;
    const int ti = 16 * Bk + 8 * th + pp;
    const int c0 = 32 * cq + 8 * a4, cb = cq >> 1, ca = 4 * (cq & 1) + a4;
    const uint32_t toff = cb * CBT + swz(ti, ca);
    auto ftab = [&](int row, float (&f)[8]) {
        const float *src = FT + row * FSTRIDE + c0;
        const float4 u0 = *(const float4 *)src, u1 = *(const float4 *)(src + 4);
        f[0] = u0.x; f[1] = u0.y; f[2] = u0.z; f[3] = u0.w; f[4] = u1.x; f[5] = u1.y; f[6] = u1.z; f[7] = u1.w;
    };
    // pass A's results for pass C (this thread's token and channels)
    float yq[8], yk[8], yv[8], Gh[8];

    // ============================================================ passes A and B of chunk nn
    // Chunk n + 1's run while the tensor pipe executes chunk n's state update; they write the
    // factor table, beta, exp(G_C), the masks and the norm partials, all consumed by chunk n
    // before that, and read chunk n's raw tiles (the conv history), which stay until the load
    // of chunk n + 2.  False when the wait for the tiles gave up.
    auto prep_ab = [&](int nn) -> bool {
        const int X = nn & 1;
        const uint8_t *stg = sm + (X ? OFF_STG1 : OFF_STG0);
        const uint8_t *prv = sm + (X ? OFF_STG0 : OFF_STG1);
        const int t0 = nn * CK;
        mbar_wait_bounded(&bar_tma[X], (uint32_t)((nn >> 1) & 1), abort_flag, p.err, p.wait_ns);
        if (tid < CK) {
            cp_async_wait_all();
            const int t = t0 + tid;
            const uint32_t wv = BRAW[(nn & 1) * CK + tid];
            const bool hi = t < T && (((uintptr_t)(p.b + (size_t)(row0 + t) * p.H + h)) & 2);
            BETAsm[tid] = sigmoid_fast(__uint_as_float(hi ? (wv & 0xffff0000u) : (wv << 16)));
            if (nn + 1 < nchunks) b_async(nn + 1);
        }
        const int nvalid = T - t0;
        // short conv + SiLU: y[c] = SiLU(sum_u w[c][u] x[i - 3 + u][c]); rows before the chunk
        // come from the previous chunk's tile, or are zero at the sequence start
        auto conv = [&](int st_off, int tensor, float (&y)[8]) {
            float x[4][8];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int r = ti - 3 + u;
                if (r >= 0) unpack8(*(const uint4 *)(stg + st_off + cb * CBT + swz(r, ca)), x[u]);
                else if (nn > 0) unpack8(*(const uint4 *)(prv + st_off + cb * CBT + swz(r + CK, ca)), x[u]);
                else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[u][e] = 0.0f;
                }
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float4 w = *(const float4 *)(CW + (tensor * DD + c0 + e) * 4);
                float acc = w.x * x[0][e];
                acc = fmaf(w.y, x[1][e], acc);
                acc = fmaf(w.z, x[2][e], acc);
                acc = fmaf(w.w, x[3][e], acc);
                y[e] = silu_fast(acc);
            }
        };
        conv(ST_Q, 0, yq);
        conv(ST_K, 1, yk);
        conv(ST_V, 2, yv);
        float sq = 0.0f, sk = 0.0f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            sq += yq[e] * yq[e];
            sk += yk[e] * yk[e];
        }
        sq += __shfl_xor_sync(0xffffffffu, sq, 8);
        sq += __shfl_xor_sync(0xffffffffu, sq, 16);
        sk += __shfl_xor_sync(0xffffffffu, sk, 8);
        sk += __shfl_xor_sync(0xffffffffu, sk, 16);
        if (a4 == 0) {
            NRM[cq * CK + ti] = sq;
            NRM[4 * CK + cq * CK + ti] = sk;
        }
        // gate; rows past the sequence's end enter with g = 0 (no decay), as the prefill's
        // zero-filled tiles do
        {
            float x[8];
            unpack8(*(const uint4 *)(stg + ST_G + toff), x);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float gv = fmaxf(-gscale * softplus_fast(x[e] + DTB[c0 + e]), p.g_lb);
                Gh[e] = ti < nvalid ? gv : 0.0f;
            }
        }
        // in-half inclusive prefix by an 8-lane scan; the last lane publishes the half sums
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            float l = Gh[e];
            float y = __shfl_up_sync(0xffffffffu, l, 1, 8);
            if (pp >= 1) l += y;
            y = __shfl_up_sync(0xffffffffu, l, 2, 8);
            if (pp >= 2) l += y;
            y = __shfl_up_sync(0xffffffffu, l, 4, 8);
            if (pp >= 4) l += y;
            Gh[e] = l;
        }
        if (pp == 7) {
            float *dst = FT + (FT_HS + 2 * Bk + th) * FSTRIDE + c0;
            *(float4 *)dst = make_float4(Gh[0], Gh[1], Gh[2], Gh[3]);
            *(float4 *)(dst + 4) = make_float4(Gh[4], Gh[5], Gh[6], Gh[7]);
        }
        __syncthreads();
        if (*abort_flag) return false;   // the wait for this chunk's tiles gave up
        tma_consumed = nn + 1;
        // pass B, one (block, channel) per thread of the first 256: block log-decays and
        //   fG = exp(G_blockstart), fL = exp(G_C - G_blockend), fM = exp(-L_B / 2) / SC (1 / SC for
        //   a block below BAD_LOG: block-start reference), fC = exp(m_1 - G_end of block 0)
        if (tid < 2 * DD) {
            const int c = tid & (DD - 1), Bq = tid >> 7;
            const float L0 = FT[FT_HS * FSTRIDE + c] + FT[(FT_HS + 1) * FSTRIDE + c];
            const float L1 = FT[(FT_HS + 2) * FSTRIDE + c] + FT[(FT_HS + 3) * FSTRIDE + c];
            const float L = Bq ? L1 : L0;
            const bool badB = !(L >= BAD_LOG);
            FT[(FT_G + Bq) * FSTRIDE + c] = __expf(Bq ? L0 : 0.0f);
            FT[(FT_L + Bq) * FSTRIDE + c] = __expf(Bq ? 0.0f : L1);
            FT[(FT_M + Bq) * FSTRIDE + c] = __expf((badB ? 0.0f : -0.5f * L) - LN_SC);
            if (badB) atomicOr(&badmask[Bq * 4 + (c >> 5)], 1u << (c & 31));
            if (Bq == 0) {
                FT[FT_C * FSTRIDE + c] = __expf(L1 >= BAD_LOG ? 0.5f * L1 : 0.0f);
                GCsm[c] = __expf(L0 + L1);
            }
        }
        // the previous chunk's output store must have read its staging tile before this
        // chunk's tiles are replaced by the load after next
        if (tid == 0) bulk_wait_read_all();
        __syncthreads();
        return true;
    };

    // The q/k value and the log-decay of one (token, channel) of the current chunk, recomputed
    // from the raw tiles for the exact diagonal path (rare: channels with a block log-decay below
    // BAD_LOG).
    auto qk_at = [&](const uint8_t *stg, const uint8_t *prv, bool first, int t, int c, bool is_q) -> float {
        const int st_off = is_q ? ST_Q : ST_K;
        const int tensor = is_q ? 0 : 1;
        float x[4];
        for (int u = 0; u < 4; ++u) {
            const int r = t - 3 + u;
            const int cc = c & 63, off_c = (c >> 6) * CBT + 2 * (cc & 7);
            x[u] = 0.0f;
            if (r >= 0) x[u] = __bfloat162float(*(const __nv_bfloat16 *)(stg + st_off + off_c + swz(r, cc >> 3)));
            else if (!first) x[u] = __bfloat162float(*(const __nv_bfloat16 *)(prv + st_off + off_c + swz(r + CK, cc >> 3)));
        }
        const float4 w = *(const float4 *)(CW + (tensor * DD + c) * 4);
        float acc = w.x * x[0];
        acc = fmaf(w.y, x[1], acc);
        acc = fmaf(w.z, x[2], acc);
        acc = fmaf(w.w, x[3], acc);
        const float y = silu_fast(acc);
        const float *nr = NRM + (is_q ? 0 : 4 * CK);
        return y * rsqrtf(nr[t] + nr[CK + t] + nr[2 * CK + t] + nr[3 * CK + t] + L2_EPS);
    };
    auto g_at = [&](const uint8_t *stg, int t, int c, int nvalid) -> float {
        if (t >= nvalid) return 0.0f;
        const int cc = c & 63;
        const float x = __bfloat162float(*(const __nv_bfloat16 *)(stg + ST_G + (c >> 6) * CBT + swz(t, cc >> 3) + 2 * (cc & 7)));
        return fmaxf(-gscale * softplus_fast(x + DTB[c]), p.g_lb);
    };

    bool alive = nchunks > 0 && prep_ab(0);
    for (int n = 0; alive && n < nchunks; ++n) {
        const int X = n & 1;
        uint8_t *stg = sm + (X ? OFF_STG1 : OFF_STG0);
        const uint8_t *prv = sm + (X ? OFF_STG0 : OFF_STG1);
        const int t0 = n * CK;
        const int nvalid = T - t0;
        const bool tail = PACKED && nvalid < CK;

        // ============================================================ pass C
        {
            const float *nq = NRM, *nk = NRM + 4 * CK;
            const float rq = rsqrtf(nq[ti] + nq[CK + ti] + nq[2 * CK + ti] + nq[3 * CK + ti] + L2_EPS);
            const float rk = rsqrtf(nk[ti] + nk[CK + ti] + nk[2 * CK + ti] + nk[3 * CK + ti] + L2_EPS);
            float qf[8], kf[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                qf[e] = yq[e] * rq;
                kf[e] = ti < nvalid ? yk[e] * rk : 0.0f;   // rows past the end add nothing
            }
            // exact diagonal of P: q_i . k_i, summed over the quarter's 4 lanes here
            float pd = 0.0f;
#pragma unroll
            for (int e = 0; e < 8; ++e) pd += qf[e] * kf[e];
            pd += __shfl_xor_sync(0xffffffffu, pd, 8);
            pd += __shfl_xor_sync(0xffffffffu, pd, 16);
            if (a4 == 0) PDsm[cq * CK + ti] = pd;
            // E1 = SC exp(G_i - G_blockstart), E2 = SC exp(G_blockend - G_i)
            float h0[8], h1[8], E1[8], E2[8], f[8], o[8];
            ftab(FT_HS + 2 * Bk, h0);
            ftab(FT_HS + 2 * Bk + 1, h1);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float gin = Gh[e] + (th ? h0[e] : 0.0f);
                E1[e] = __expf(gin + LN_SC);
                E2[e] = __expf(h0[e] + h1[e] - gin + LN_SC);
            }
            uint4 hi, lo;
            // Q^ = Gamma q, K^ = Gamma k with Gamma = exp(G_i) = (E1 / SC) fG
            ftab(FT_G + Bk, f);
            float gam[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                gam[e] = (E1[e] * INV_SC) * f[e];
                o[e] = qf[e] * gam[e];
            }
            split8(o, hi, lo);
            *(uint4 *)(sm + OFF_QK + cb * QK_CB + swz(ti, ca)) = hi;
            *(uint4 *)(sm + OFF_QL + toff) = lo;
#pragma unroll
            for (int e = 0; e < 8; ++e) o[e] = kf[e] * gam[e];
            *(uint4 *)(sm + OFF_QK + cb * QK_CB + QK_K + swz(ti, ca)) = pack8(o);
            // K~ = exp(G_C - G_i) k = k (E2 / SC) fL
            ftab(FT_L + Bk, f);
#pragma unroll
            for (int e = 0; e < 8; ++e) o[e] = kf[e] * ((E2[e] * INV_SC) * f[e]);
            split8(o, hi, lo);
            *(uint4 *)(sm + OFF_KTH + toff) = hi;
            *(uint4 *)(sm + OFF_KTL + toff) = lo;
            // V
            split8(yv, hi, lo);
            *(uint4 *)(sm + OFF_VH + toff) = hi;
            *(uint4 *)(sm + OFF_VL + toff) = lo;
            // Gram rows [Q_B; K_B] scaled by E1 fM = exp(G_i - m_B)
            ftab(FT_M + Bk, f);
            const int rq_row = 32 * Bk + 8 * th + pp;
            {
                float rf[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    rf[e] = E1[e] * f[e];
                    o[e] = qf[e] * rf[e];
                }
                split8(o, hi, lo);
                *(uint4 *)(gr + GR_RH + cb * R_CB + swz(rq_row, ca)) = hi;
                *(uint4 *)(gr + GR_RL + cb * R_CB + swz(rq_row, ca)) = lo;
#pragma unroll
                for (int e = 0; e < 8; ++e) o[e] = kf[e] * rf[e];
                split8(o, hi, lo);
                *(uint4 *)(gr + GR_RH + cb * R_CB + swz(rq_row + 16, ca)) = hi;
                *(uint4 *)(gr + GR_RL + cb * R_CB + swz(rq_row + 16, ca)) = lo;
            }
            // Gram columns, own block: k E2 fM = k exp(m_B - G_j) (0 for channels below BAD_LOG,
            // added exactly after the readback)
            const uint32_t badbits = (badmask[Bk * 4 + (c0 >> 5)] >> (c0 & 31)) & 0xffu;
#pragma unroll
            for (int e = 0; e < 8; ++e) o[e] = (badbits >> e & 1u) ? 0.0f : kf[e] * (E2[e] * f[e]);
            split8(o, hi, lo);
            *(uint4 *)(gr + GR_CV + cb * CV_CB + swz(ti, ca)) = hi;
            *(uint4 *)(gr + GR_CV + cb * CV_CB + CV_LO + swz(ti, ca)) = lo;
            // Gram columns of block 0's tokens for block 1's rows: k (E2 / SC) fC
            if (Bk == 0) {
                ftab(FT_C, f);
#pragma unroll
                for (int e = 0; e < 8; ++e) o[e] = kf[e] * ((E2[e] * INV_SC) * f[e]);
                split8(o, hi, lo);
                *(uint4 *)(gr + GR_CV + cb * CV_CB + swz(CK + ti, ca)) = hi;
                *(uint4 *)(gr + GR_CV + cb * CV_CB + CV_LO + swz(CK + ti, ca)) = lo;
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        if (*abort_flag) break;   // the previous chunk's state wait gave up

        // ============================================================ Gram: R_hi [CV_hi; CV_lo] (N = 96) + R_lo CV_hi
        if (tid == 0) {
            tc_fence_after();
            const uint32_t sRH = smem_u32(gr + GR_RH), sRL = smem_u32(gr + GR_RL), sCV = smem_u32(gr + GR_CV);
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t orr = (kk >> 2) * R_CB + (kk & 3) * 32, oc = (kk >> 2) * CV_CB + (kk & 3) * 32;
                mma_ss(tmem + TM_G, sdesc(sRH + orr, 16, 1024), sdesc(sCV + oc, 16, 1024), id_gram96, kk > 0);
                mma_ss(tmem + TM_G, sdesc(sRL + orr, 16, 1024), sdesc(sCV + oc, 16, 1024), id_gram, 1);
            }
            mma_commit(bar_mma);
        }
        mma_wait();
        tc_fence_after();

        // ============================================================ readback -> P (hi, lo), A
        if (lq < 2) {
            // lane quarter lq = row block: lanes 0..15 its P rows (q side), 16..31 its A rows;
            // column group cg = 8-column chunk m of j.  Block 1's earlier columns sit at D
            // columns 32.., the own block's at the token index.
            const int B = lq, m = cg;
            const bool is_q = lane < 16;
            const int i = 16 * B + (lane & 15);
            const float bi = BETAsm[i];
            const float pdiag = (PDsm[i] + PDsm[CK + i]) + (PDsm[2 * CK + i] + PDsm[3 * CK + i]);
            const int dcol = B == 0 ? (m < 2 ? 8 * m : -1) : (m < 2 ? CK + 8 * m : 8 * m);
            uint32_t r[8], r2[8];
            if (dcol >= 0) {
                tmem_ld8(tmem + lane_q + TM_G + dcol, r);
                tmem_ld8(tmem + lane_q + TM_G + 48 + dcol, r2);   // the R_hi CV_lo term
                tmem_wait_ld();
            }
            float vals[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int j = 8 * m + e;
                const float v = dcol >= 0 ? __uint_as_float(r[e]) + __uint_as_float(r2[e]) : 0.0f;
                vals[e] = is_q ? (j < i ? v : (j == i ? pdiag : 0.0f)) : (j < i ? bi * v : 0.0f);
            }
            // exact own-block terms of channels below BAD_LOG, recomputed from the raw tiles
            // (rare path)
            const uint32_t *bmask = badmask + 4 * B;
            for (int wd = 0; wd < 4; ++wd) {
                for (uint32_t mk = bmask[wd]; mk != 0u; mk &= mk - 1u) {
                    const int c = 32 * wd + __ffs((int)mk) - 1;
                    const float xi = (t0 + i < T) ? qk_at(stg, prv, n == 0, i, c, is_q) : 0.0f;
                    float w = 1.0f;   // exp(G_i - G_j), built backwards from j = i
                    for (int j = i; j >= 16 * B; --j) {
                        if (j < i && (j >> 3) == m) {
                            const float kj = (t0 + j < T) ? qk_at(stg, prv, n == 0, j, c, false) : 0.0f;
                            vals[j & 7] += (is_q ? 1.0f : bi) * xi * kj * w;
                        }
                        w *= __expf(g_at(stg, j, c, nvalid));
                    }
                }
            }
            if (is_q) {
                uint4 hi, lo;
                split8(vals, hi, lo);
                *(uint4 *)(gr + GR_PH + swz(i, m)) = hi;
                *(uint4 *)(gr + GR_PL + swz(i, m)) = lo;
            } else {
                *(float4 *)(A32 + i * AST + 8 * m) = make_float4(vals[0], vals[1], vals[2], vals[3]);
                *(float4 *)(A32 + i * AST + 8 * m + 4) = make_float4(vals[4], vals[5], vals[6], vals[7]);
            }
        }
        __syncthreads();
        if (*abort_flag) break;   // the Gram wait gave up
        if (tid < 8) badmask[tid] = 0u;   // consumed
        if (tid == 0 && n + 1 < nchunks) {
            // the other stage held chunk n - 1: its raw rows (the conv history of the exact path
            // above) are no longer read and its output store has read its staging tile
            bulk_wait_read_all();
            issue_tma(n + 1);
        }

        // ============================================================ T (warp 0) || Y, O init (warps 8..15)
        if (warp == 0) {
            // T = (I + A)^{-1} Diag(beta): lane j solves column j of L = I + A in its registers,
            // left-looking: x_i = -sum_{m < i} A[i][m] x_m for i > j, x_j = 1.  Every lane reads
            // the same row segment of A (a broadcast); the loops unroll completely.  All fp32.
            const int j = lane;
            float x[CK];
#pragma unroll
            for (int i = 0; i < CK; ++i) x[i] = i == j ? 1.0f : 0.0f;
#pragma unroll
            for (int i = 1; i < CK; ++i) {
                float acc0 = 0.0f, acc1 = 0.0f;
#pragma unroll
                for (int m4 = 0; m4 < i; m4 += 4) {
                    const float4 av = *(const float4 *)(A32 + i * AST + m4);
                    acc0 = fmaf(av.x, x[m4], acc0);
                    if (m4 + 1 < i) acc1 = fmaf(av.y, x[m4 + 1], acc1);
                    if (m4 + 2 < i) acc0 = fmaf(av.z, x[m4 + 2], acc0);
                    if (m4 + 3 < i) acc1 = fmaf(av.w, x[m4 + 3], acc1);
                }
                x[i] = i == j ? 1.0f : -(acc0 + acc1);
            }
            // T hi, lo in bf16, K-major [i][j]; above the diagonal x is zero
            const float bj = BETAsm[j];
#pragma unroll
            for (int i = 0; i < CK; ++i) {
                const float tv = x[i] * bj;
                const __nv_bfloat16 th_ = __float2bfloat16_rn(tv);
                const uint32_t o = swz(i, j >> 3) + 2 * (j & 7);
                *(__nv_bfloat16 *)(gr + GR_TH + o) = th_;
                *(__nv_bfloat16 *)(gr + GR_TL + o) = __float2bfloat16_rn(tv - __bfloat162float(th_));
            }
            fence_proxy_async();
        } else if (warp >= 8) {
            const int hb = (warp - 8) >> 2;   // column half of the state this warp splits
            // S^T (fp32, key channels 64 hb ..) -> bf16 hi + lo for the Y and O-init MMAs, which
            // read only these copies, so the state is decayed by exp(G_C) in the same pass
#pragma unroll
            for (int cc = 0; cc < 64; cc += 32) {
                uint32_t r[32], hi[16], lo[16];
                const uint32_t ta = tmem + lane_q + TM_S + 64 * hb + cc;
                tmem_ld32(ta, r);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float x0 = __uint_as_float(r[2 * e]), x1 = __uint_as_float(r[2 * e + 1]);
                    hi[e] = pack_bf16x2(x0, x1);
                    const float2 hv = unpack_bf16x2(hi[e]);
                    lo[e] = pack_bf16x2(x0 - hv.x, x1 - hv.y);
                }
                tmem_st16(tmem + lane_q + TM_SH + 32 * hb + cc / 2, hi);
                tmem_st16(tmem + lane_q + TM_SL + 32 * hb + cc / 2, lo);
#pragma unroll
                for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * GCsm[64 * hb + cc + e]);
                tmem_st32(ta, r);
            }
            tmem_wait_st();
            tc_fence_before();
            named_bar_sync(2, 256);
            if (tid == 256) {
                // [O^T | Y^T] = S^T [Q^_hi; K^]^T from S_hi and S_lo (N = 64), then O^T += S_hi Q^_lo
                tc_fence_after();
                const uint32_t sQK = smem_u32(sm + OFF_QK), sQL = smem_u32(sm + OFF_QL);
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t oqk = (kk >> 2) * QK_CB + (kk & 3) * 32, oql = (kk >> 2) * CBT + (kk & 3) * 32;
                    mma_ts(tmem + TM_O, tmem + TM_SH + kk * 8, sdesc(sQK + oqk, 16, 1024), id_n64, kk > 0);
                    mma_ts(tmem + TM_O, tmem + TM_SL + kk * 8, sdesc(sQK + oqk, 16, 1024), id_n64, 1);
                    mma_ts(tmem + TM_O, tmem + TM_SH + kk * 8, sdesc(sQL + oql, 16, 1024), id_n32, 1);
                }
                mma_commit(bar_y);
                mma_commit(bar_oi);
            }
            if (mbar_wait_bounded(bar_y, (uint32_t)(n & 1), abort_flag, p.err, p.wait_ns)) {
                tc_fence_after();
                // Y^T (fp32, tokens 16 hb ..) -> bf16 hi + lo
                uint32_t r[16], hi[8], lo[8];
                tmem_ld16(tmem + lane_q + TM_Y + 16 * hb, r);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float x0 = __uint_as_float(r[2 * e]), x1 = __uint_as_float(r[2 * e + 1]);
                    hi[e] = pack_bf16x2(x0, x1);
                    const float2 hv = unpack_bf16x2(hi[e]);
                    lo[e] = pack_bf16x2(x0 - hv.x, x1 - hv.y);
                }
                tmem_st8(tmem + lane_q + TM_HI + 8 * hb, hi);
                tmem_st8(tmem + lane_q + TM_LO + 8 * hb, lo);
                tmem_wait_st();
            }
            mbar_wait_bounded(bar_oi, (uint32_t)(n & 1), abort_flag, p.err, p.wait_ns);
        }
        tc_fence_before();
        __syncthreads();
        if (*abort_flag) break;

        // ============================================================ U^T = V^T T^T - Y^T T^T (hi/lo pairs)
        if (tid == 0) {
            tc_fence_after();
            const uint32_t sVH = smem_u32(sm + OFF_VH), sVL = smem_u32(sm + OFF_VL);
            const uint32_t sTH = smem_u32(gr + GR_TH), sTL = smem_u32(gr + GR_TL);
            for (int kk = 0; kk < 2; ++kk) {
                const uint64_t tH = sdesc(sTH + kk * 32, 16, 1024), tL = sdesc(sTL + kk * 32, 16, 1024);
                mma_ss(tmem + TM_U, sdesc(sVH + kk * 2048, CBT, 1024), tH, id_v, kk > 0);
                mma_ss(tmem + TM_U, sdesc(sVL + kk * 2048, CBT, 1024), tH, id_v, 1);
                mma_ss(tmem + TM_U, sdesc(sVH + kk * 2048, CBT, 1024), tL, id_v, 1);
                mma_ts(tmem + TM_U, tmem + TM_HI + kk * 8, tH, id_n32_neg, 1);
                mma_ts(tmem + TM_U, tmem + TM_LO + kk * 8, tH, id_n32_neg, 1);
                mma_ts(tmem + TM_U, tmem + TM_HI + kk * 8, tL, id_n32_neg, 1);
            }
            mma_commit(bar_mma);
        }
        mma_wait();
        tc_fence_after();
        if (cg < 2) {
            // U^T fp32 (tokens 16 cg ..) -> bf16 hi, lo (Y's copies are consumed)
            uint32_t r[16], hi[8], lo[8];
            tmem_ld16(tmem + lane_q + TM_U + 16 * cg, r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float x0 = __uint_as_float(r[2 * e]), x1 = __uint_as_float(r[2 * e + 1]);
                hi[e] = pack_bf16x2(x0, x1);
                const float2 hv = unpack_bf16x2(hi[e]);
                lo[e] = pack_bf16x2(x0 - hv.x, x1 - hv.y);
            }
            tmem_st8(tmem + lane_q + TM_HI + 8 * cg, hi);
            tmem_st8(tmem + lane_q + TM_LO + 8 * cg, lo);
            tmem_wait_st();
        }
        tc_fence_before();
        __syncthreads();
        if (*abort_flag) break;   // the U wait gave up

        // ============================================================ O += U P,  S^T += U^T K~
        if (tid == 0) {
            tc_fence_after();
            const uint32_t sPH = smem_u32(gr + GR_PH), sPL = smem_u32(gr + GR_PL);
            const uint32_t sKH = smem_u32(sm + OFF_KTH), sKL = smem_u32(sm + OFF_KTL);
            for (int kk = 0; kk < 2; ++kk) {
                mma_ts(tmem + TM_O, tmem + TM_HI + kk * 8, sdesc(sPH + kk * 32, 16, 1024), id_n32, 1);
                mma_ts(tmem + TM_O, tmem + TM_LO + kk * 8, sdesc(sPH + kk * 32, 16, 1024), id_n32, 1);
                mma_ts(tmem + TM_O, tmem + TM_HI + kk * 8, sdesc(sPL + kk * 32, 16, 1024), id_n32, 1);
            }
            mma_commit(bar_o);
            for (int kk = 0; kk < 2; ++kk) {
                mma_ts(tmem + TM_S, tmem + TM_HI + kk * 8, sdesc(sKH + kk * 2048, CBT, 1024), id_s, 1);
                mma_ts(tmem + TM_S, tmem + TM_LO + kk * 8, sdesc(sKH + kk * 2048, CBT, 1024), id_s, 1);
                mma_ts(tmem + TM_S, tmem + TM_HI + kk * 8, sdesc(sKL + kk * 2048, CBT, 1024), id_s, 1);
            }
            mma_commit(bar_mma);
        }

        // ============================================================ epilogue: RMSNorm x gain x sigmoid gate
        mbar_wait_bounded(bar_o, (uint32_t)(n & 1), abort_flag, p.err, p.wait_ns);
        tc_fence_after();
        {
            // thread: value column v = 32 lq + lane, tokens 8 cg .. 8 cg + 7
            const int v = 32 * lq + lane;
            uint32_t r[8];
            tmem_ld8(tmem + lane_q + TM_O + 8 * cg, r);
            tmem_wait_ld();
            float o[8], ss[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                o[e] = __uint_as_float(r[e]);
                ss[e] = o[e] * o[e];
            }
            // sums over the warp's 32 value columns of the 8 tokens by a reduce-scatter: after
            // the xor-16, -8 and -4 steps lane l holds token (l >> 2) & 7's partial over 8 lanes,
            // the xor-2 and -1 steps complete it
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const bool up = lane & 16;
                const float send = up ? ss[k] : ss[4 + k];
                ss[k] = (up ? ss[4 + k] : ss[k]) + __shfl_xor_sync(0xffffffffu, send, 16);
            }
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const bool up = lane & 8;
                const float send = up ? ss[k] : ss[2 + k];
                ss[k] = (up ? ss[2 + k] : ss[k]) + __shfl_xor_sync(0xffffffffu, send, 8);
            }
            {
                const bool up = lane & 4;
                const float send = up ? ss[0] : ss[1];
                ss[0] = (up ? ss[1] : ss[0]) + __shfl_xor_sync(0xffffffffu, send, 4);
            }
            ss[0] += __shfl_xor_sync(0xffffffffu, ss[0], 2);
            ss[0] += __shfl_xor_sync(0xffffffffu, ss[0], 1);
            if ((lane & 3) == 0) RMS[lq * CK + 8 * cg + ((lane >> 2) & 7)] = ss[0];
            __syncthreads();
            const float gain = GAIN[v];
            const uint32_t vo = (v >> 6) * CBT + 2 * (v & 7);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int i = 8 * cg + e;
                const float ms = (RMS[i] + RMS[CK + i]) + (RMS[2 * CK + i] + RMS[3 * CK + i]);
                const float rr = rsqrtf(ms / (float)DD + p.eps);
                const float y = __bfloat162float(__float2bfloat16_rn(o[e] * rr)) * gain;   // cast to bf16, then gain
                const uint32_t eo = vo + swz(i, (v & 63) >> 3);
                const float zv = __bfloat162float(*(const __nv_bfloat16 *)(stg + ST_Z + eo));
                *(__nv_bfloat16 *)(stg + ST_G + eo) = __float2bfloat16_rn(y * sigmoid_fast(zv));
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        if (*abort_flag) break;   // the O wait gave up
        if (tail) {
            // the last chunk of a packed sequence: only its valid rows are written
            for (int u = tid; u < CK * 16; u += NT) {
                const int i = u >> 4, j = u & 15;
                if (i < nvalid)
                    *(uint4 *)(p.out + ((size_t)(row0 + t0 + i) * p.H + h) * DD + 8 * j) =
                        *(const uint4 *)(stg + ST_G + (j >> 3) * CBT + swz(i, j & 7));
            }
        } else if (tid == 0) {
            tma_store_4d(&tm_o, stg + ST_G, 0, h, tt0 + t0, tb);
            tma_store_4d(&tm_o, stg + ST_G + CBT, 64, h, tt0 + t0, tb);
            bulk_commit();
        }
        // the next chunk's passes A and B run while the tensor pipe updates the state
        if (n + 1 < nchunks && !prep_ab(n + 1)) break;
        mma_wait();   // checked after the next barrier, before the next chunk's Gram issue
        tc_fence_after();
    }

    // ---------------------------------------------------------------- final state
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (p.sT && !*abort_flag) {
        const int v = 32 * lq + lane;
        float *sT = p.sT + (size_t)bh * DD * DD;
        uint32_t r[32];
        tmem_ld32(tmem + lane_q + TM_S + 32 * cg, r);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) sT[(size_t)(32 * cg + e) * DD + v] = __uint_as_float(r[e]);
    }
    if (*abort_flag) {
        // a bounded wait gave up: everything asynchronous this CTA started finishes before its
        // shared and tensor memory are released (see chunk_tc.cu)
        constexpr unsigned long long DRAIN_NS = 2000000000ull;
        if (tid == 0 || tid == 256) mma_commit(bar_drain);
        if (tid == 0) {
            if (tma_issued > tma_consumed) {
                const int c = tma_consumed;
                mbar_wait_timed(&bar_tma[c & 1], (uint32_t)((c >> 1) & 1), DRAIN_NS);
            }
            mbar_wait_timed(bar_drain, 0u, DRAIN_NS);
        }
    }
    if (tid < CK) cp_async_wait_all();
    if (tid == 0) bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace

bool layer_tc_supported(const LayerTcArgs &a)
{
    return a.io == IO_BF16 && a.dk == DD && a.dv == DD && a.T > 0 && ((uintptr_t)a.b_raw & 3) == 0 &&
           device_is_sm100() && tensor_maps_available();
}

cudaError_t launch_layer_tc(const LayerTcArgs &a, cudaStream_t s)
{
    CUtensorMap mq, mk, mv, mg, mz, mo;
    const int mb = a.cu ? 1 : a.B;
    if (!make_tile_map(&mq, a.q_raw, mb, a.T, a.H, CK) || !make_tile_map(&mk, a.k_raw, mb, a.T, a.H, CK) ||
        !make_tile_map(&mv, a.v_raw, mb, a.T, a.H, CK) || !make_tile_map(&mg, a.g_raw, mb, a.T, a.H, CK) ||
        !make_tile_map(&mz, a.o_gate_raw, mb, a.T, a.H, CK) || !make_tile_map(&mo, a.out, mb, a.T, a.H, CK))
        return cudaErrorInvalidValue;
    struct TagFixed;
    struct TagPacked;
    cudaError_t e = smem_opt_in<TagFixed>((const void *)kda_layer_tc_kernel<false>, SMEM_BYTES);
    if (e == cudaSuccess) e = smem_opt_in<TagPacked>((const void *)kda_layer_tc_kernel<true>, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const WaitHooks hk = wait_hooks();
    LayerTcParams p{(const __nv_bfloat16 *)a.q_raw, (const __nv_bfloat16 *)a.k_raw, (const __nv_bfloat16 *)a.g_raw,
                    (const __nv_bfloat16 *)a.b_raw, a.conv_q, a.conv_k, a.conv_v, a.A_log, a.dt_bias, a.gain,
                    a.g_lb, a.eps, a.s0, a.sT, (__nv_bfloat16 *)a.out, a.T, a.H, a.err, a.cu,
                    hk.wait_ns, hk.skip_load_chunk};
    if (a.cu) kda_layer_tc_kernel<true><<<a.B * a.H, NT, SMEM_BYTES, s>>>(mq, mk, mv, mg, mz, mo, p);
    else kda_layer_tc_kernel<false><<<a.B * a.H, NT, SMEM_BYTES, s>>>(mq, mk, mv, mg, mz, mo, p);
    return cudaGetLastError();
}

}  // namespace kda
