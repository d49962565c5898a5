// chunk_tc.cu — chunked KDA prefill on tcgen05 tensor cores (bf16 I/O, dk = dv = 128).
//
// One CTA owns one (b, h) head and walks its chunks of C = 64 tokens in order.  The
// fp32 state lives in tensor memory for the whole sequence, transposed (lane = value
// column v, column = key channel c).  Per chunk, with G_i = sum_{s<=i} g_s (per channel)
// and blocks of 16 tokens inside the chunk:
//
//   prep (CUDA cores)   per-(block, channel) decay factors, then Q^ = Gamma*Q (fp32),
//                       K^ = Gamma*K, K~ = exp(G_C - G)*K and the Gram operands (below).
//   Gram (tcgen05)      [Q;K] rows x CV_I columns -> P (j <= i) and A' (j < i) in one
//                       M=128, N=160, K=128 MMA, plus a residual MMA for the diagonal blocks.
//   inverse (CUDA)      T = (I + Diag(beta) A')^{-1} Diag(beta), blocked, fp32 — while the
//                       tensor cores compute O^T = S^T Q^^T and Y^T = S^T K^^T.
//   U (tcgen05)         U^T = V^T T^T - Y^T T^T, i.e. U = T (V - K^ S).
//   chain (tcgen05)     O^T += U^T P^T;  S^T <- S^T Diag(exp G_C) + U^T K~.
// The product that reads the state for the output (S^T Q^^T) runs as a kind::tf32 MMA with
// the fp32 state itself as the TMEM A operand; Y = K^ S uses the state split into bf16
// hi + lo parts.
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
// second MMA with the rounding residuals (R_lo CVd + R CVd_lo), U, Y, P and K~ enter their
// products as hi + lo bf16 pairs (O += U_hi P_hi + U_lo P_hi + U_hi P_lo,
// S += K~_hi^T (U_hi + U_lo) + K~_lo^T U_hi), and the state is read at tf32 precision from
// its fp32 copy for S^T Q^^T (Q^ kept in fp32).
#include <cuda.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace kda {
namespace {

using namespace tc;

constexpr int NT = 512;       // threads: 16 warps = 4 TMEM lane quarters x 4 column groups
constexpr int CK = 64;        // chunk
constexpr int DD = 128;       // dk = dv
constexpr float BAD_LOG = -168.0f;  // block log-decays below this take the exact fallback

// shared memory layout (offsets from a 1024-byte aligned base)
constexpr int REG_BYTES = 73728;                 // 72 KB: stage (q,k,v,g) or Gram operands
constexpr int OFF_REG0 = 0;
constexpr int OFF_REG1 = REG_BYTES;
constexpr int ST_Q = 0, ST_K = 16384, ST_V = 32768, ST_G = 49152;     // inside a stage region
constexpr int GR_R = 0, GR_CV = 32768;                                // inside a Gram region
// K~ lo (bf16 MN-major, one 64-channel block per region): channel block cb lives at offset
// ST_KLO of region cb, past the stage tiles.  In chunk n the stage region (n & 1) has that
// tail free from the load onwards, so its block is written during prep; the other region's
// tail holds Gram columns until the Gram MMA has run, so that block waits in tensor memory
// (the U columns, unused until the U MMA) and is copied there after the Gram.  Both are read
// by the state-update MMA at the chunk's end.
constexpr int ST_KLO = 65536;
constexpr int R_CB = 16384;                      // R: 128 rows x 128 B per channel block
constexpr int CV_ROWS = 160, CV_CB = CV_ROWS * 128;
// X1 (32 KB): Q^ in fp32 (tf32 K-major [i][c]), from prep until the O-init MMA (issued
// after the Gram readback) has run
// X2 (32 KB): R_lo (prep -> Gram); then A and L^{-1} in fp32 (inverse)
// P and P_lo (bf16 K-major [i][j], 8 KB each) take the stage's q tile once the Gram MMAs have
// read the residual columns kept there; T (bf16 K-major [i][j], 8 KB) sits in the factor
// table; the O tile is staged in the stage's V tile
constexpr int OFF_X1 = 2 * REG_BYTES;
constexpr int OFF_QH = OFF_X1;                   // 32 KB: 4 K-blocks of 32 fp32 x 64 rows
constexpr int ST_P = ST_Q, ST_PL = ST_Q + 8192;  // inside the stage region
constexpr int OFF_X2 = OFF_X1 + 32768;
// A and L^{-1}: fp32 [64][AST]; the row stride of 68 floats shifts consecutive rows by four
// banks, so column reads and row-segment writes spread over all banks.  L^{-1} runs 2 KB past
// X2 into the factor table, which is dead between prep and the next chunk.
constexpr int AST = 68;
constexpr int OFF_A32 = OFF_X2;
constexpr int OFF_LINV = OFF_X2 + 64 * AST * 4;
// per-(block, channel) table, fp32 rows of FSTRIDE (128 channels + padding that puts the
// four blocks of one channel in different banks): fG, fL, fM for blocks 0..3, the half-block
// log-decays (row FT_HS + 2 B + half: sum of g over tokens 8 half .. 8 half + 7 of block B),
// then fC for the six (B, I) pairs with I > B
constexpr int FSTRIDE = 136;
constexpr int FT_G = 0, FT_L = 4, FT_M = 8, FT_HS = 12, FT_C = 20;   // row numbers
constexpr int FT_BYTES = 26 * FSTRIDE * 4;
constexpr int OFF_FT = OFF_X2 + 32768;
constexpr int OFF_T = OFF_FT + 2048;             // past L^{-1}'s overhang, 1024-aligned
constexpr int OFF_MISC = OFF_FT + FT_BYTES;
constexpr int MS_BADMASK = 0;                    // uint32 [4][4]: channels with L_B < BAD_LOG, per block
constexpr int MS_GC = 64;                        // fp32 [128] chunk decay exp(G_C)
constexpr int MS_BETA = 576;                     // fp32 [64]
constexpr int MS_PD = 832;                       // fp32 [4][64]: exact q_i . k_i, per channel quarter
constexpr int MS_BAR = 1856;                     // uint64 [5]: tma0, tma1, mma, O init, Y
constexpr int MS_TSLOT = 1896;                   // uint32
constexpr int MS_ABORT = 1900;                   // int
constexpr int MS_DRAIN = 1904;                   // uint64: MMA drain after an abort
constexpr int MS_BRAW = 1920;                    // uint32 [2][64]: beta words in flight (cp.async)
constexpr int MS_BAROC = 2432;                   // uint64: the chunk's O MMAs
constexpr int MISC_BYTES = 2448;
constexpr int SMEM_BYTES = OFF_MISC + MISC_BYTES + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory per block");
static_assert(OFF_LINV + 64 * AST * 4 <= OFF_MISC, "L^{-1} stays clear of the barriers");
static_assert(OFF_MISC % 16 == 0 && OFF_FT % 16 == 0 && OFF_T % 1024 == 0 && OFF_T + 8192 <= OFF_MISC, "alignment");
__host__ __device__ constexpr int fc_slot(int B, int I) { return B == 0 ? I - 1 : (B == 1 ? I + 1 : 5); }
KDA_DEVICE int aidx(int i, int j) { return i * AST + j; }

// tensor memory columns
constexpr uint32_t TM_S = 0;       // fp32 S^T, 128 cols
constexpr uint32_t TM_G = 128;     // Gram D, 160 cols; after the Gram readback:
constexpr uint32_t TM_SH = 128;    //   bf16 S^T hi (A operand), 64 cols
constexpr uint32_t TM_SL = 192;    //   bf16 S^T lo, 64 cols
constexpr uint32_t TM_HI32 = 256;  //   bf16 Y^T hi, then U^T hi (A operands), 32 cols
constexpr uint32_t TM_U = 288;     // U^T, 64 cols
constexpr uint32_t TM_O = 352;     // O^T, 64 cols
constexpr uint32_t TM_CORR = 416;  // diagonal-block Gram correction R_lo CVd + R CVd_lo, 64 cols
constexpr uint32_t TM_Y = 416;     //   then Y^T = S^T K^^T, 64 cols
constexpr uint32_t TM_LO32 = 480;  // bf16 Y^T lo, then U^T lo, 32 cols

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
    const int *cu;   // packed variable length: sequence offsets (null: fixed length T)
    unsigned long long wait_ns;   // limit of each bounded mbarrier wait
    int skip_load_chunk;          // failure injection: this chunk's tile load is never issued (-1: none)
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

// PACKED: N sequences of different lengths back to back (offsets p.cu), one batch row of the
// tensor maps; otherwise B sequences of T tokens.  The fixed-length instance carries none of
// the packed bookkeeping.
template <bool PACKED>
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
    uint32_t *BRAW = (uint32_t *)(misc + MS_BRAW);
    uint64_t *bar_tma = (uint64_t *)(misc + MS_BAR);
    uint64_t *bar_mma = bar_tma + 2;
    uint64_t *bar_o = bar_tma + 3;
    uint64_t *bar_y = bar_tma + 4;
    uint32_t *tslot = (uint32_t *)(misc + MS_TSLOT);
    volatile int *abort_flag = (volatile int *)(misc + MS_ABORT);
    uint64_t *bar_drain = (uint64_t *)(misc + MS_DRAIN);
    uint64_t *bar_oc = (uint64_t *)(misc + MS_BAROC);
    float *A32 = (float *)(sm + OFF_A32);
    float *LINV = (float *)(sm + OFF_LINV);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x, b = bh / p.H, h = bh % p.H;
    // this sequence's tokens: rows row0 .. row0 + T - 1 of the flattened token axis; the 4-D
    // tensor maps address them as (token tt0 + t, batch tb)
    const SeqSpan span = PACKED ? seq_span(p.cu, b, p.T) : SeqSpan{b * p.T, p.T};
    const int T = span.len, row0 = span.row0;
    const int tt0 = PACKED ? row0 : 0, tb = PACKED ? 0 : b;
    const int nchunks = (T + CK - 1) / CK;
    // a warp reaches TMEM lanes 32 (warp & 3) .. + 31; the four warps of a lane quarter split
    // the columns of every TMEM tile they read or write into column groups cg = warp >> 2
    const int lq = warp & 3, cg = warp >> 2;
    const uint32_t lane_q = (uint32_t)(32 * lq) << 16;

    if (tid == 0) {
        mbar_init(&bar_tma[0], 1);
        mbar_init(&bar_tma[1], 1);
        mbar_init(bar_mma, 1);
        mbar_init(bar_o, 1);
        mbar_init(bar_y, 1);
        mbar_init(bar_oc, 1);
        mbar_init(bar_drain, 3);   // the three MMA-issuing threads
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

    // Loads issued by thread 0 and loads consumed (uniform: counted after the barrier that
    // follows the wait); after an abort at most one issued load has not been waited for.
    int tma_issued = 0, tma_consumed = 0;
    auto issue_tma = [&](int n) {
        if (n == p.skip_load_chunk) return;   // injected failure: the wait for it runs out
        ++tma_issued;
        const int r = n & 1;
        uint8_t *st = sm + (r ? OFF_REG1 : OFF_REG0);
        const int t0 = tt0 + n * CK;
        mbar_arrive_expect_tx(&bar_tma[r], 4 * 16384);
        for (int cb = 0; cb < 2; ++cb) {
            tma_load_4d(st + ST_Q + cb * 8192, &tm_q, cb * 64, h, t0, tb, &bar_tma[r]);
            tma_load_4d(st + ST_K + cb * 8192, &tm_k, cb * 64, h, t0, tb, &bar_tma[r]);
            tma_load_4d(st + ST_V + cb * 8192, &tm_v, cb * 64, h, t0, tb, &bar_tma[r]);
            tma_load_4d(st + ST_G + cb * 8192, &tm_g, cb * 64, h, t0, tb, &bar_tma[r]);
        }
    };
    if (tid == 0 && nchunks > 0) issue_tma(0);

    // ---------------------------------------------------------------- initial state
    {
        // S^T: lane v = value column, TMEM column c = key channel
        const int v = 32 * lq + lane;
        const float *s0 = p.s0 ? p.s0 + (size_t)bh * DD * DD : nullptr;
        uint32_t r[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(s0 ? s0[(size_t)(32 * cg + e) * DD + v] : 0.0f);
        tmem_st32(tmem + lane_q + TM_S + 32 * cg, r);
        tmem_wait_st();
    }

    uint32_t mma_phase = 0;
    // A wait that gives up sets *abort_flag (and the device error word); every thread then
    // leaves the chunk loop at the next check of the flag, each placed right after a block
    // barrier and before any TMA or MMA issue, so the decision is the same for the whole CTA.
    auto mma_wait = [&]() {
        mbar_wait_bounded(bar_mma, mma_phase, abort_flag, p.err, p.wait_ns);
        mma_phase ^= 1u;
    };

    constexpr uint32_t id_gram = idesc_bf16(128, CV_ROWS, false, false);
    constexpr uint32_t id_corr = idesc_bf16(128, 64, false, false);
    constexpr uint32_t id_o0 = idesc_tf32(128, 64, false, false);
    constexpr uint32_t id_wt = idesc_bf16(128, 64, true, false);
    constexpr uint32_t id_opn = idesc_bf16(128, 64, false, false, true);
    constexpr uint32_t id_op = idesc_bf16(128, 64, false, false);
    constexpr uint32_t id_s = idesc_bf16(128, 128, false, true);
    constexpr uint32_t id_s64 = idesc_bf16(128, 64, false, true);

    // beta of the next chunk is copied one chunk ahead, global -> shared by cp.async, so no
    // thread ever waits on its memory latency: the aligned 32-bit word that holds beta_t
    // (2 bytes of it when beta_t is the word's low half, which may be the last element)
    auto beta_async = [&](int nn) {   // tid < CK
        const int t = nn * CK + tid;
        const void *src = p.beta;
        uint32_t bytes = 0;
        if (t < T) {
            const uintptr_t ea = (uintptr_t)(p.beta + (size_t)(row0 + t) * p.H + h);
            bytes = (ea & 2) ? 4u : 2u;
            src = (const void *)(ea & ~(uintptr_t)3);
        }
        cp_async4(smem_u32(BRAW + (nn & 1) * CK + tid), src, bytes);
        cp_async_commit();
    };
    if (tid < CK && nchunks > 0) beta_async(0);

    for (int n = 0; n < nchunks; ++n) {
        const int X = n & 1;
        uint8_t *stg = sm + (X ? OFF_REG1 : OFF_REG0);
        uint8_t *gro = sm + (X ? OFF_REG0 : OFF_REG1);
        const int t0 = n * CK;

        mbar_wait_bounded(&bar_tma[X], (uint32_t)((n >> 1) & 1), abort_flag, p.err, p.wait_ns);

        // ============================================================ prep
        if (tid < CK) {
            cp_async_wait_all();
            const int t = t0 + tid;
            const uint32_t wv = BRAW[(n & 1) * CK + tid];
            const bool hi = t < T && (((uintptr_t)(p.beta + (size_t)(row0 + t) * p.H + h)) & 2);
            BETAsm[tid] = __uint_as_float(hi ? (wv & 0xffff0000u) : (wv << 16));
            if (n + 1 < nchunks) beta_async(n + 1);
        }
        constexpr float INV_SC = 7.523164e-37f;    // SC = 2^120, INV_SC = 2^-120
        constexpr float LN_SC = 83.17766f;         // 120 ln 2
        // Token mapping of passes A and C: warp (pr, cq, th) takes token position pp = lane & 7
        // of the half th of block pr (s = 0) and of block 3 - pr (s = 1), so every warp carries
        // the same number of later-block Gram columns; lane >> 3 picks 8 of the 32 channels of
        // quarter cq.
        const int pr = warp & 1;
        const int cq = (warp >> 1) & 3;   // channel quarter (32 channels)
        const int th = warp >> 3;         // token half of the block
        const int pp = lane & 7;          // token position inside the half
        const int a = 4 * (cq & 1) + (lane >> 3);   // 16-byte chunk inside the channel block
        const int cb = cq >> 1;           // channel block (64 channels)
        const int c0 = 64 * cb + 8 * a;
        auto ftab = [&](int row, float (&f)[8]) {
            const float *src = FT + row * FSTRIDE + c0;
            const float4 u0 = *(const float4 *)src, u1 = *(const float4 *)(src + 4);
            f[0] = u0.x; f[1] = u0.y; f[2] = u0.z; f[3] = u0.w; f[4] = u1.x; f[5] = u1.y; f[6] = u1.z; f[7] = u1.w;
        };
        // Rows at or past the end of a packed sequence (the next sequence's tokens) enter as
        // g = 0 and k = 0: they then add nothing to the decays, A, P's columns, Y or the state
        // update, and their own output rows are not stored.  (Fixed length: the tensor maps'
        // zero fill past T does the same.)
        const int nvalid = T - t0;
        const bool tail = PACKED && nvalid < CK;   // the same for the whole block
        // pass A: in-half inclusive prefix of g by an 8-lane scan; the last lane of each half
        // publishes the half-block sums
        float Gh[2][8];
#pragma unroll
        for (int s = 0; s < 2; ++s) {
            const int B = s == 0 ? pr : 3 - pr;
            const int i = 16 * B + 8 * th + pp;
            unpack8(*(const uint4 *)(stg + ST_G + cb * 8192 + swz(i, a)), Gh[s]);
            if (tail && i >= nvalid) {
#pragma unroll
                for (int e = 0; e < 8; ++e) Gh[s][e] = 0.0f;
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                float l = Gh[s][e];
                float y = __shfl_up_sync(0xffffffffu, l, 1, 8);
                if (pp >= 1) l += y;
                y = __shfl_up_sync(0xffffffffu, l, 2, 8);
                if (pp >= 2) l += y;
                y = __shfl_up_sync(0xffffffffu, l, 4, 8);
                if (pp >= 4) l += y;
                Gh[s][e] = l;
            }
            if (pp == 7) {
                float *dst = FT + (FT_HS + 2 * B + th) * FSTRIDE + c0;
                *(float4 *)dst = make_float4(Gh[s][0], Gh[s][1], Gh[s][2], Gh[s][3]);
                *(float4 *)(dst + 4) = make_float4(Gh[s][4], Gh[s][5], Gh[s][6], Gh[s][7]);
            }
        }
        __syncthreads();
        if (*abort_flag) break;   // the wait for this chunk's tiles gave up
        tma_consumed = n + 1;
        // pass B, one (block, channel) per thread: block log-decays L_J and the factors
        //   fG = exp(G_blockstart)      fL = exp(G_C - G_blockend)
        //   fM = exp(-L_B / 2) / SC     (block-start reference, 1 / SC, where L_B < BAD_LOG)
        //   fC(B, I) = exp(m_I - G_blockend of B) for later blocks I > B, m_I the reference of I.
        // All exponents are sums of non-positive log-decays (plus L_B / 2 >= -84 for fM), so a
        // factor underflows only where the exact value does.
        {
            const int c = tid & 127, Bq = tid >> 7;
            float Lv[4];
#pragma unroll
            for (int J = 0; J < 4; ++J) Lv[J] = FT[(FT_HS + 2 * J) * FSTRIDE + c] + FT[(FT_HS + 2 * J + 1) * FSTRIDE + c];
            float lpre = 0.0f, lpost = 0.0f, L = 0.0f;
#pragma unroll
            for (int J = 0; J < 4; ++J) {
                if (J < Bq) lpre += Lv[J];
                if (J > Bq) lpost += Lv[J];
                if (J == Bq) L = Lv[J];
            }
            const bool badB = !(L >= BAD_LOG);
            float *ft = FT + Bq * FSTRIDE + c;
            ft[FT_G * FSTRIDE] = __expf(lpre);
            ft[FT_L * FSTRIDE] = __expf(lpost);
            ft[FT_M * FSTRIDE] = __expf((badB ? 0.0f : -0.5f * L) - LN_SC);
            if (badB) atomicOr(&badmask[Bq * 4 + (c >> 5)], 1u << (c & 31));
#pragma unroll
            for (int I = 1; I < 4; ++I) {
                if (I <= Bq) continue;
                float l = Lv[I] >= BAD_LOG ? 0.5f * Lv[I] : 0.0f;
#pragma unroll
                for (int J = 1; J < 3; ++J)
                    if (J > Bq && J < I) l += Lv[J];
                FT[(FT_C + fc_slot(Bq, I)) * FSTRIDE + c] = __expf(l);
            }
            if (Bq == 0) GCsm[c] = __expf(Lv[0] + Lv[1] + Lv[2] + Lv[3]);
        }
        // the previous chunk's O tile (its stage region takes this chunk's Gram operands in pass
        // C) must have been read out by its TMA store, and its state-update MMAs, which read K~
        // hi and lo where pass C writes the Gram operands, must have completed (they ran under
        // the O staging, the store and passes A and B)
        if (tid == 0) bulk_wait_read_all();
        if (n > 0) mma_wait();
        __syncthreads();
        // pass C, per token.  With SC = 2^120:
        //   E1 = SC exp(G_i - G_blockstart)  (includes token i)
        //   E2 = SC exp(G_blockend - G_i)    (excludes token i)
        // from log-domain prefix sums, so no partial product can underflow; both are normal
        // numbers for block log-decays down to BAD_LOG (SC e^-168 ~ e^-84.8).
        uint32_t klo[8];   // this thread's K~ lo, two tokens x 8 channels of channel block cb
        {
#pragma unroll
            for (int s = 0; s < 2; ++s) {
                const int B = s == 0 ? pr : 3 - pr;
                const int i = 16 * B + 8 * th + pp;
                const uint32_t off = cb * 8192 + swz(i, a);
                float Gin[8], Lb[8];
                {
                    // G_i - G_blockstart = in-half prefix (+ the first half's sum); L_B
                    float h0[8], h1[8];
                    ftab(FT_HS + 2 * B, h0);
                    ftab(FT_HS + 2 * B + 1, h1);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        Gin[e] = Gh[s][e] + (th ? h0[e] : 0.0f);
                        Lb[e] = h0[e] + h1[e];
                    }
                }
                const uint32_t badbits = (badmask[B * 4 + (c0 >> 5)] >> (c0 & 31)) & 0xffu;
                float qf[8], kf[8], o[8], E1[8], E2[8], f[8];
                unpack8(*(const uint4 *)(stg + ST_Q + off), qf);
                unpack8(*(const uint4 *)(stg + ST_K + off), kf);
                if (tail && i >= nvalid) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) kf[e] = 0.0f;
                }
                // exact diagonal of P: partial q_i . k_i over this lane's 8 channels, summed over
                // the quarter's 4 lanes
                float pd = 0.0f;
#pragma unroll
                for (int e = 0; e < 8; ++e) pd += qf[e] * kf[e];
                pd += __shfl_xor_sync(0xffffffffu, pd, 8);
                pd += __shfl_xor_sync(0xffffffffu, pd, 16);
                if (lane < 8) PDsm[cq * CK + i] = pd;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    E1[e] = __expf(Gin[e] + LN_SC);
                    E2[e] = __expf(Lb[e] - Gin[e] + LN_SC);
                }
                // Q^ = Gamma q (fp32 K-major tile for the tf32 MMA), Gamma_i = (E1 / SC) fG
                ftab(FT_G + B, f);
                float gam[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    gam[e] = (E1[e] * INV_SC) * f[e];
                    o[e] = qf[e] * gam[e];
                }
                {
                    uint8_t *qh = sm + OFF_QH + (2 * cb + (a >> 2)) * 8192;
                    *(float4 *)(qh + swz(i, 2 * (a & 3))) = make_float4(o[0], o[1], o[2], o[3]);
                    *(float4 *)(qh + swz(i, 2 * (a & 3) + 1)) = make_float4(o[4], o[5], o[6], o[7]);
                }
                // K^ = Gamma k (in place)
#pragma unroll
                for (int e = 0; e < 8; ++e) o[e] = kf[e] * gam[e];
                *(uint4 *)(stg + ST_K + off) = pack8(o);
                // K~ = exp(G_C - G_i) k = k (E2 / SC) fL: bf16 hi over g, bf16 residual to the
                // K~ lo tile (now if this channel block's tail is free, else after the Gram)
                ftab(FT_L + B, f);
#pragma unroll
                for (int e = 0; e < 8; ++e) o[e] = kf[e] * ((E2[e] * INV_SC) * f[e]);
                {
                    const uint4 hk = pack8(o);
                    float hf[8], lo[8];
                    unpack8(hk, hf);
#pragma unroll
                    for (int e = 0; e < 8; ++e) lo[e] = o[e] - hf[e];
                    *(uint4 *)(stg + ST_G + off) = hk;
                    const uint4 kl = pack8(lo);
                    if (cb == X) *(uint4 *)(stg + ST_KLO + swz(i, a)) = kl;
                    klo[4 * s + 0] = kl.x; klo[4 * s + 1] = kl.y; klo[4 * s + 2] = kl.z; klo[4 * s + 3] = kl.w;
                }
                // Gram rows [Q_B; K_B] scaled by E1 fM = exp(G_i - m_B): hi part to the Gram
                // rows, bf16 residual to X2 (free until the readback)
                ftab(FT_M + B, f);
                const int rq = 32 * B + 8 * th + pp;
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
                // Gram columns, diagonal block: k E2 fM = k exp(m_B - G_j), 0 for channels with
                // L_B < BAD_LOG (those terms are added exactly after the readback); hi part to
                // diagonal column row i, bf16 residual over the (now dead) raw q
                {
                    float hf[8], lo[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) o[e] = (badbits >> e & 1u) ? 0.0f : kf[e] * (E2[e] * f[e]);
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
                    ftab(FT_C + fc_slot(B, I), f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) o[e] = kf[e] * ((E2[e] * INV_SC) * f[e]);
                    *(uint4 *)(gro + GR_CV + cb * CV_CB + swz(cv_off(I) + i, a)) = pack8(o);
                }
            }
        }
        // the half of K~ lo whose region tail still holds Gram columns waits in the U columns
        // (8 per thread of this lane quarter, column group warp >> 2)
        if (cb != X) tmem_st8(tmem + lane_q + TM_U + 8 * (warp >> 2), klo);
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        if (*abort_flag) break;   // the previous chunk's state-update wait gave up

        // ============================================================ Gram (MMA)
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
            mma_commit(bar_mma);
        }
        mma_wait();
        tc_fence_after();
        if (tid == 0 && n + 1 < nchunks && !*abort_flag) {
            // the Gram region is free now; it was the stage of chunk n - 1, whose O tile must
            // have been read out by its TMA store.  (If another thread's wait gave up, the abort
            // path waits for this load before the CTA exits.)
            bulk_wait_read_all();
            issue_tma(n + 1);
        }
        if (cb != X) {
            // the Gram MMA has read the other region's tail: this channel block's K~ lo goes there
            uint32_t r[8];
            tmem_wait_st();
            tmem_ld8(tmem + lane_q + TM_U + 8 * (warp >> 2), r);
            tmem_wait_ld();
#pragma unroll
            for (int s = 0; s < 2; ++s)
                *(uint4 *)(gro + ST_KLO + swz(16 * (s == 0 ? pr : 3 - pr) + 8 * th + pp, a)) =
                    make_uint4(r[4 * s], r[4 * s + 1], r[4 * s + 2], r[4 * s + 3]);
            fence_proxy_async();
        }

        // ============================================================ Gram readback -> P, A
        {
            // lanes 0..15 of lane quarter I: P rows (q side), lanes 16..31: A rows (k side).
            // CV_I has 2 (I + 1) chunks of 8 columns; chunk m goes to column group m % 4.
            const int I = lq;
            const bool is_q = lane < 16;
            const int i = 16 * I + (lane & 15);
            const int nch = 2 * (I + 1);
            const float bi = BETAsm[i];
            const float pdiag = (PDsm[i] + PDsm[CK + i]) + (PDsm[2 * CK + i] + PDsm[3 * CK + i]);   // exact q_i . k_i
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
                    *(uint4 *)(stg + ST_P + swz(i, j0 >> 3)) = hi;
                    *(uint4 *)(stg + ST_PL + swz(i, j0 >> 3)) = pack8(lo);
                } else {
                    *(float4 *)(A32 + aidx(i, j0)) = make_float4(vals[0], vals[1], vals[2], vals[3]);
                    *(float4 *)(A32 + aidx(i, j0 + 4)) = make_float4(vals[4], vals[5], vals[6], vals[7]);
                }
            };
            uint32_t r[2][8], c8[2][8];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int m = cg + 4 * u;
                if (m < 2 * I) {
                    tmem_ld8(tmem + lane_q + TM_G + cv_off(I) + 8 * m, r[u]);   // earlier blocks
                } else if (m < nch) {
                    tmem_ld8(tmem + lane_q + TM_G + 8 * m, r[u]);               // own (diagonal) block
                    tmem_ld8(tmem + lane_q + TM_CORR + 8 * m, c8[u]);
                }
            }
            tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int m = cg + 4 * u;
                if (m < nch) {
                    if (m >= 2 * I) {
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            r[u][e] = __float_as_uint(__uint_as_float(r[u][e]) + __uint_as_float(c8[u][e]));
                    }
                    emit(8 * m, r[u]);
                } else if (is_q) {
                    // P is an MMA operand: its upper part must be zero (A's is never read)
                    *(uint4 *)(stg + ST_P + swz(i, m)) = make_uint4(0, 0, 0, 0);
                    *(uint4 *)(stg + ST_PL + swz(i, m)) = make_uint4(0, 0, 0, 0);
                }
            }
            // exact diagonal-block terms of channels whose block decay underflows the Gram
            // factorisation, added in place to this thread's own entries (rare path)
            const uint32_t *bmask = badmask + 4 * I;
            for (int wd = 0; wd < 4; ++wd) {
                for (uint32_t mk = bmask[wd]; mk != 0u; mk &= mk - 1u) {
                    const int c = 32 * wd + __ffs((int)mk) - 1;
                    const size_t rowi = ((size_t)(row0 + t0 + i) * p.H + h) * DD + c;
                    const float xi = (t0 + i < T) ? __bfloat162float((is_q ? p.q : p.k)[rowi]) : 0.0f;
                    float w = 1.0f;   // exp(G_i - G_j), built backwards from j = i
                    for (int j = i; j >= 16 * I; --j) {
                        const bool valid = t0 + j < T;
                        const size_t rowj = ((size_t)(row0 + t0 + j) * p.H + h) * DD + c;
                        if (j < i && ((j >> 3) & 3) == cg) {
                            const float d = xi * (valid ? __bfloat162float(p.k[rowj]) : 0.0f) * w;
                            if (is_q) {
                                __nv_bfloat16 *ph = (__nv_bfloat16 *)(stg + ST_P + swz(i, j >> 3)) + (j & 7);
                                __nv_bfloat16 *pl = (__nv_bfloat16 *)(stg + ST_PL + swz(i, j >> 3)) + (j & 7);
                                const float v = __bfloat162float(*ph) + __bfloat162float(*pl) + d;
                                const __nv_bfloat16 vh = __float2bfloat16_rn(v);
                                *ph = vh;
                                *pl = __float2bfloat16_rn(v - __bfloat162float(vh));
                            } else {
                                A32[aidx(i, j)] += bi * d;
                            }
                        }
                        w *= __expf(valid ? __bfloat162float(p.g[rowj]) : 0.0f);
                    }
                }
            }
        }
        __syncthreads();
        if (*abort_flag) break;   // the Gram wait gave up
        if (tid < 16) badmask[tid] = 0u;   // masks consumed
        // ============================================================ T (warps 0..7) || Y = K^ S (warps 8..15)
        // Warps 0..7 invert L = I + A and form T (named barrier 1).  Warps 8..15 (named barrier
        // 2) issue the O init, split the chunk-start state S^T into bf16 hi + lo in tensor
        // memory, issue Y^T = S^T K^^T (one bf16 MMA chain per part, fp32 accumulate), split
        // Y^T the same way and decay the state by exp(G_C).  After both:  U^T = V^T T^T - Y_hi^T T^T - Y_lo^T T^T, i.e.
        // U = T (V - K^ S) = U~ - W S, with S entering at about 2^-16 relative precision.
        if (warp < 8) {
            // L = I + A, inverted in two levels of 2x2 blocks.  16x16 diagonal inverses
            // L_II^{-1} by right-looking forward substitution (one column per thread); then each
            // 32x32 half  [[L_a, 0], [A_ba, L_b]]^{-1} = [[L_a^{-1}, 0], [-L_b^{-1} A_ba L_a^{-1}, L_b^{-1}]]
            // and the same rule once more for the 64x64 matrix with 32x32 blocks.  Every product
            // is a full-precision fp32 dot product (16x16 blocks: one output per thread and
            // half; 32x32 blocks: 4 rows x 1 column per thread).  Scratch (P, Q) lives in A's
            // unused upper-right 32x32 block.
            if (tid < 64) {
                const int Ib = tid >> 4, col = tid & 15;
                float x[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) x[r] = r == col ? 1.0f : 0.0f;
#pragma unroll
                for (int m = 0; m < 15; ++m)
#pragma unroll
                    for (int r = m + 1; r < 16; ++r) x[r] -= A32[aidx(16 * Ib + r, 16 * Ib + m)] * x[m];
#pragma unroll
                for (int r = 0; r < 16; ++r) LINV[aidx(16 * Ib + r, 16 * Ib + col)] = x[r];
            }
            named_bar_sync(1, 256);
            // dot16(X, xr, xc, Y, yr, yc): sum_m X[xr][xc + m] Y[yr + m][yc], m < 16
            auto dot16 = [&](const float *Xm, int xr, int xc, const float *Ym, int yr, int yc) -> float {
                float s0 = 0.0f, s1 = 0.0f;
#pragma unroll
                for (int m4 = 0; m4 < 16; m4 += 4) {
                    const float4 xv = *(const float4 *)(Xm + aidx(xr, xc + m4));
                    s0 += xv.x * Ym[aidx(yr + m4 + 0, yc)] + xv.z * Ym[aidx(yr + m4 + 2, yc)];
                    s1 += xv.y * Ym[aidx(yr + m4 + 1, yc)] + xv.w * Ym[aidx(yr + m4 + 3, yc)];
                }
                return s0 + s1;
            };
            {
                // halves h = 0 (blocks 0, 1) and h = 1 (blocks 2, 3):
                // P_h = A_{2h+1,2h} L_{2h}^{-1}  ->  scratch rows 0..15, columns 32 + 16 h ..
                const int r = tid >> 4, c = tid & 15;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
                    A32[aidx(r, 32 + 16 * hh + c)] = dot16(A32, 32 * hh + 16 + r, 32 * hh, LINV, 32 * hh, 32 * hh + c);
                named_bar_sync(1, 256);
                // T_{2h+1,2h} = -L_{2h+1}^{-1} P_h; the (2h, 2h+1) block is zero
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int ra = 32 * hh, rb = ra + 16;
                    LINV[aidx(rb + r, ra + c)] = -dot16(LINV, rb + r, rb, A32, 0, 32 + 16 * hh + c);
                    LINV[aidx(ra + r, rb + c)] = 0.0f;
                }
                named_bar_sync(1, 256);
            }
            {
                // Q = A_{[2,3],[0,1]} L_{[0,1]}^{-1}: 4 rows x 1 column per thread
                const int c = tid & 31, rg = tid >> 5;   // rows 4 rg .. 4 rg + 3 of 32
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int m4 = 0; m4 < 32; m4 += 4) {
                    float y[4];
#pragma unroll
                    for (int t = 0; t < 4; ++t) y[t] = LINV[aidx(m4 + t, c)];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float4 xv = *(const float4 *)(A32 + aidx(32 + 4 * rg + q, m4));
                        acc[q] += xv.x * y[0] + xv.y * y[1] + xv.z * y[2] + xv.w * y[3];
                    }
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) A32[aidx(4 * rg + q, 32 + c)] = acc[q];
                named_bar_sync(1, 256);
                // T_{[2,3],[0,1]} = -L_{[2,3]}^{-1} Q
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[q] = 0.0f;
#pragma unroll
                for (int m4 = 0; m4 < 32; m4 += 4) {
                    float y[4];
#pragma unroll
                    for (int t = 0; t < 4; ++t) y[t] = A32[aidx(m4 + t, 32 + c)];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float4 xv = *(const float4 *)(LINV + aidx(32 + 4 * rg + q, 32 + m4));
                        acc[q] += xv.x * y[0] + xv.y * y[1] + xv.z * y[2] + xv.w * y[3];
                    }
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) LINV[aidx(32 + 4 * rg + q, c)] = -acc[q];
                named_bar_sync(1, 256);
            }
#pragma unroll
            for (int it = 0; it < 2; ++it) {
                // T = L^{-1} Diag(beta), lower triangle, bf16 K-major [i][j]
                const int idx = tid + 256 * it, i = idx >> 3, jc = idx & 7;
                const float4 l0 = *(const float4 *)(LINV + aidx(i, 8 * jc)), l1 = *(const float4 *)(LINV + aidx(i, 8 * jc + 4));
                const float4 b0 = *(const float4 *)(BETAsm + 8 * jc), b1 = *(const float4 *)(BETAsm + 8 * jc + 4);
                const float lv[8] = {l0.x, l0.y, l0.z, l0.w, l1.x, l1.y, l1.z, l1.w};
                const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
                float vals[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) vals[e] = 8 * jc + e <= i ? lv[e] * bv[e] : 0.0f;
                *(uint4 *)(sm + OFF_T + swz(i, jc)) = pack8(vals);
            }
            fence_proxy_async();
        } else {
            const int hb = (warp - 8) >> 2;   // column half of the TMEM tiles this warp splits
            if (tid == NT - 32) {
                // O^T = S^T Q^^T at tf32 (A = fp32 state in TMEM, 8 key channels per MMA); it
                // completes on bar_o before the state is decayed
                tc_fence_after();
                const uint32_t sQ = smem_u32(sm + OFF_QH);
                for (int kk = 0; kk < 16; ++kk)
                    mma_ts_tf32(tmem + TM_O, tmem + TM_S + kk * 8, sdesc(sQ + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024),
                                id_o0, kk > 0);
                mma_commit(bar_o);
            }
            // S^T (fp32, key channels 64 hb .. 64 hb + 63) -> bf16 hi + lo, two per column
#pragma unroll
            for (int cc = 0; cc < 64; cc += 32) {
                uint32_t r[32], hi[16], lo[16];
                tmem_ld32(tmem + lane_q + TM_S + 64 * hb + cc, r);
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
            }
            tmem_wait_st();
            tc_fence_before();
            named_bar_sync(2, 256);
            if (tid == 256) {
                // Y^T = S_hi^T K^^T + S_lo^T K^^T  (K^ = Gamma k, bf16 K-major in the stage)
                tc_fence_after();
                const uint32_t sK = smem_u32(stg + ST_K);
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tmem + TM_Y, tmem + TM_SH + kk * 8, sdesc(sK + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024),
                           id_op, kk > 0);
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tmem + TM_Y, tmem + TM_SL + kk * 8, sdesc(sK + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024),
                           id_op, 1);
                mma_commit(bar_y);
            }
            if (mbar_wait_bounded(bar_y, (uint32_t)(n & 1), abort_flag, p.err, p.wait_ns)) {
                tc_fence_after();
                // Y^T (fp32, tokens 32 hb .. 32 hb + 31) -> bf16 hi + lo
                uint32_t r[32], hi[16], lo[16];
                tmem_ld32(tmem + lane_q + TM_Y + 32 * hb, r);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float x0 = __uint_as_float(r[2 * e]), x1 = __uint_as_float(r[2 * e + 1]);
                    hi[e] = pack_bf16x2(x0, x1);
                    const float2 hv = unpack_bf16x2(hi[e]);
                    lo[e] = pack_bf16x2(x0 - hv.x, x1 - hv.y);
                }
                tmem_st16(tmem + lane_q + TM_HI32 + 16 * hb, hi);
                tmem_st16(tmem + lane_q + TM_LO32 + 16 * hb, lo);
                tmem_wait_st();
            }
            // S^T <- S^T Diag(exp G_C): every reader of the chunk-start state is done once the
            // O init has completed (the split above and the Y MMAs read the copies)
            if (mbar_wait_bounded(bar_o, (uint32_t)(n & 1), abort_flag, p.err, p.wait_ns)) {
                tc_fence_after();
#pragma unroll
                for (int cc = 0; cc < 64; cc += 32) {
                    uint32_t sr[32];
                    const uint32_t ta = tmem + lane_q + TM_S + 64 * hb + cc;
                    tmem_ld32(ta, sr);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) sr[e] = __float_as_uint(__uint_as_float(sr[e]) * GCsm[64 * hb + cc + e]);
                    tmem_st32(ta, sr);
                }
                tmem_wait_st();
            }
        }
        tc_fence_before();
        __syncthreads();
        if (*abort_flag) break;

        // ============================================================ U^T = V^T T^T - Y_hi^T T^T - Y_lo^T T^T
        if (tid == 0) {
            tc_fence_after();
            const uint32_t sV = smem_u32(stg + ST_V), sT_ = smem_u32(sm + OFF_T);
            for (int kk = 0; kk < 4; ++kk)
                mma_ss(tmem + TM_U, sdesc(sV + kk * 2048, 8192, 1024), sdesc(sT_ + kk * 32, 16, 1024), id_wt, kk > 0);
            for (int kk = 0; kk < 4; ++kk)
                mma_ts(tmem + TM_U, tmem + TM_HI32 + kk * 8, sdesc(sT_ + kk * 32, 16, 1024), id_opn, 1);
            for (int kk = 0; kk < 4; ++kk)
                mma_ts(tmem + TM_U, tmem + TM_LO32 + kk * 8, sdesc(sT_ + kk * 32, 16, 1024), id_opn, 1);
            mma_commit(bar_mma);
        }
        mma_wait();
        tc_fence_after();
        {
            // U^T fp32 -> bf16 hi and lo A operands (two bf16 per 32-bit column; Y's are consumed)
            uint32_t r[16], r8[8], l8[8];
            tmem_ld16(tmem + lane_q + TM_U + 16 * cg, r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float x0 = __uint_as_float(r[2 * e]), x1 = __uint_as_float(r[2 * e + 1]);
                r8[e] = pack_bf16x2(x0, x1);
                const float2 hv = unpack_bf16x2(r8[e]);
                l8[e] = pack_bf16x2(x0 - hv.x, x1 - hv.y);
            }
            tmem_st8(tmem + lane_q + TM_HI32 + 8 * cg, r8);
            tmem_st8(tmem + lane_q + TM_LO32 + 8 * cg, l8);
            tmem_wait_st();
        }
        tc_fence_before();
        __syncthreads();
        if (*abort_flag) break;   // the U wait gave up
        if (tid == 0) {
            tc_fence_after();
            const uint32_t sP = smem_u32(stg + ST_P), sPL = smem_u32(stg + ST_PL), sG = smem_u32(stg + ST_G);
            const uint32_t sKL0 = smem_u32(sm + OFF_REG0 + ST_KLO), sKL1 = smem_u32(sm + OFF_REG1 + ST_KLO);
            for (int kk = 0; kk < 4; ++kk) {
                mma_ts(tmem + TM_O, tmem + TM_HI32 + kk * 8, sdesc(sP + kk * 32, 16, 1024), id_op, 1);
                mma_ts(tmem + TM_O, tmem + TM_LO32 + kk * 8, sdesc(sP + kk * 32, 16, 1024), id_op, 1);
                mma_ts(tmem + TM_O, tmem + TM_HI32 + kk * 8, sdesc(sPL + kk * 32, 16, 1024), id_op, 1);
            }
            mma_commit(bar_oc);   // O is read out while the state update runs
            for (int kk = 0; kk < 4; ++kk) {
                mma_ts(tmem + TM_S, tmem + TM_HI32 + kk * 8, sdesc(sG + kk * 2048, 8192, 1024), id_s, 1);
                mma_ts(tmem + TM_S, tmem + TM_LO32 + kk * 8, sdesc(sG + kk * 2048, 8192, 1024), id_s, 1);
                // K~ lo, one 64-channel block (state columns) per MMA
                mma_ts(tmem + TM_S, tmem + TM_HI32 + kk * 8, sdesc(sKL0 + kk * 2048, 8192, 1024), id_s64, 1);
                mma_ts(tmem + TM_S + 64, tmem + TM_HI32 + kk * 8, sdesc(sKL1 + kk * 2048, 8192, 1024), id_s64, 1);
            }
            mma_commit(bar_mma);   // waited for before the next chunk's pass C (or the final state)
        }
        mbar_wait_bounded(bar_oc, (uint32_t)(n & 1), abort_flag, p.err, p.wait_ns);
        tc_fence_after();
        {
            // O^T -> bf16 tile in the stage's V tile (dead since the U~ MMA; the load tiles'
            // layout: 2 channel blocks of [64 rows x 128 B], 128-byte swizzle), then two TMA
            // stores; rows past T are clipped by the tensor map.  The stores are waited for
            // (read side) only before the next TMA load into this stage region.
            const int v = 32 * lq + lane;
            uint32_t r[16];
            tmem_ld16(tmem + lane_q + TM_O + 16 * cg, r);
            tmem_wait_ld();
            uint8_t *ot = stg + ST_V + (v >> 6) * 8192 + ((v & 7) << 1);
#pragma unroll
            for (int e = 0; e < 16; ++e)
                *(__nv_bfloat16 *)(ot + swz(16 * cg + e, (v & 63) >> 3)) = __float2bfloat16_rn(__uint_as_float(r[e]));
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        if (*abort_flag) break;   // the O wait gave up
        if (tail) {
            // the last chunk of a packed sequence: its tile's later rows are the next
            // sequence's, so only the valid rows are written, 16 bytes per thread and pass
            for (int u = tid; u < CK * 16; u += NT) {
                const int i = u >> 4, j = u & 15;
                if (i < nvalid)
                    *(uint4 *)(p.out + ((size_t)(row0 + t0 + i) * p.H + h) * DD + 8 * j) =
                        *(const uint4 *)(stg + ST_V + (j >> 3) * 8192 + swz(i, j & 7));
            }
        } else if (tid == 0) {
            tma_store_4d(&tm_o, stg + ST_V, 0, h, tt0 + t0, tb);
            tma_store_4d(&tm_o, stg + ST_V + 8192, 64, h, tt0 + t0, tb);
            bulk_commit();
        }
    }

    // ---------------------------------------------------------------- final state
    // The flag has not changed since its last check after a block barrier, so every thread
    // takes the same branch; the last chunk's state update is still running.
    if (nchunks > 0 && !*abort_flag) {
        mma_wait();
        tc_fence_after();
    }
    __syncthreads();
    if (p.sT && !*abort_flag) {
        tc_fence_after();
        const int v = 32 * lq + lane;
        float *sT = p.sT + (size_t)bh * DD * DD;
        uint32_t r[32];
        tmem_ld32(tmem + lane_q + TM_S + 32 * cg, r);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) sT[(size_t)(32 * cg + e) * DD + v] = __uint_as_float(r[e]);
    }
    if (*abort_flag) {
        // A bounded wait gave up (the flag is read after a block barrier, so the whole CTA is
        // here).  Everything asynchronous this CTA started finishes before its shared and tensor
        // memory are released: the MMAs of the three issuing threads (one commit each on
        // bar_drain), a tile load issued but not yet waited for, the beta copies and the bulk
        // stores.  These operations were really issued, so they complete; the waits are
        // bounded all the same.
        constexpr unsigned long long DRAIN_NS = 2000000000ull;
        if (tid == 0 || tid == 256 || tid == NT - 32) mma_commit(bar_drain);
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

}  // namespace

// [B, T, H, 128] bf16 -> 4-D map (128, H, T, B), box (64, 1, box_rows, 1), 128-byte swizzle,
// zero fill past T.
bool make_tile_map(CUtensorMap *m, const void *base, int B, int T, int H, int box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)DD, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)DD * 2, (cuuint64_t)H * DD * 2, (cuuint64_t)T * H * DD * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
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

bool tensor_maps_available() { return encode_fn() != nullptr; }

bool chunk_tc_supported(const ChunkArgs &a)
{
    // beta is fetched as aligned 32-bit words (cp.async), so it must start on a 4-byte boundary
    // (the entry points require 16)
    return a.io == IO_BF16 && a.dk == DD && a.dv == DD && !a.qkv_f32 && !a.g_f32 && !a.beta_f32 && !a.out_f32 &&
           a.T > 0 && ((uintptr_t)a.beta & 3) == 0 && device_is_sm100() && tensor_maps_available();
}

namespace {
std::atomic<unsigned long long> g_wait_ns{kDefaultWaitNs};
std::atomic<int> g_skip_load_chunk{-1};
}  // namespace

WaitHooks wait_hooks() { return WaitHooks{g_wait_ns.load(), g_skip_load_chunk.load()}; }

void set_wait_hooks(unsigned long long wait_ns, int skip_load_chunk)
{
    g_wait_ns.store(wait_ns ? wait_ns : kDefaultWaitNs);
    g_skip_load_chunk.store(skip_load_chunk < 0 ? -1 : skip_load_chunk);
}

cudaError_t launch_chunk_tc(const ChunkArgs &a, cudaStream_t s)
{
    CUtensorMap mq, mk, mv, mg, mo;
    const int mb = a.cu ? 1 : a.B;   // packed sequences: one batch row of all tokens
    if (!make_tile_map(&mq, a.q, mb, a.T, a.H, CK) || !make_tile_map(&mk, a.k, mb, a.T, a.H, CK) ||
        !make_tile_map(&mv, a.v, mb, a.T, a.H, CK) || !make_tile_map(&mg, a.g, mb, a.T, a.H, CK) ||
        !make_tile_map(&mo, a.out, mb, a.T, a.H, CK))
        return cudaErrorInvalidValue;
    struct TagFixed;
    struct TagPacked;
    cudaError_t attr_err = smem_opt_in<TagFixed>((const void *)kda_chunk_tc_kernel<false>, SMEM_BYTES);
    if (attr_err == cudaSuccess) attr_err = smem_opt_in<TagPacked>((const void *)kda_chunk_tc_kernel<true>, SMEM_BYTES);
    if (attr_err != cudaSuccess) return attr_err;
    const WaitHooks hk = wait_hooks();
    TcParams p{(const __nv_bfloat16 *)a.q, (const __nv_bfloat16 *)a.k, (const __nv_bfloat16 *)a.g,
               (const __nv_bfloat16 *)a.beta, a.s0, (__nv_bfloat16 *)a.out, a.sT, a.T, a.H, a.err, a.cu,
               hk.wait_ns, hk.skip_load_chunk};
    if (a.cu) kda_chunk_tc_kernel<true><<<a.B * a.H, NT, SMEM_BYTES, s>>>(mq, mk, mv, mg, mo, p);
    else kda_chunk_tc_kernel<false><<<a.B * a.H, NT, SMEM_BYTES, s>>>(mq, mk, mv, mg, mo, p);
    return cudaGetLastError();
}

}  // namespace kda
