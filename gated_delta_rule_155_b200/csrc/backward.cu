// backward.cu — gradients of the gated delta rule, chunkwise, exact fp32 on CUDA cores.
//
// The forward step per token t (per head):
//   S' = Diag(exp g_t) S;   u_t = beta_t (v_t - S'^T k_t);   S_t = S' + k_t u_t^T;   o_t = S_t^T q_t
// (the recurrence of the Kimi-K3 KDA layers; the pages' training runs differentiate it:
//  maxtext PR #5550, its jax.grad test and the C4 training steps).
//
// Chunk form over BC = 16 tokens (G = in-chunk inclusive cumsum of g, G_C its last row,
// E_ijc = exp(G_ic - G_jc) for j <= i, never above 1):
//   Abar_ij = sum_c k_ic k_jc E_ijc (j < i)      P_ij = sum_c q_ic k_jc E_ijc (j <= i)
//   M = (I + Diag(beta) Abar)^-1,  X = V - K^ S,  Z = Diag(beta) X,  U = M Z
//   O = Q^ S + P U,   S_next = Diag(exp G_C) S + K~^T U
//   with Q^ = q exp(G), K^ = k exp(G), K~ = k exp(G_C - G).
// Reverse mode through those lines, given dO and dS_next:
//   dU = P^T dO + K~ dS_next          dZ = M^T dU        dX = Diag(beta) dZ     dV = dX
//   dP = tril(dO U^T)                 dA = -stril(dZ U^T)   (since M^T dM M^T = dZ U^T)
//   dbeta = rowsum(dZ . X) + rowsum(dA . Abar),   dAbar = Diag(beta) dA
//   dq = exp(G) (dO S^T) + sum_j dP_ij k_j E_ij
//   dk = -exp(G) (dX S^T) + sum_j dAbar_ij k_j E_ij              ("+" part: G enters with +)
//      + exp(G_C - G) (U dS_next^T) + sum_m (dP_mi q_m + dAbar_mi k_m) E_mi   ("-" part)
//   dG = q dq + k dk+ - k dk-,  dG_C += sum_i k_i dk~_i + exp(G_C) rowsum(dS_next . S)
//   dg = reverse cumsum of dG;   dS = Diag(exp G_C) dS_next + Q^^T dO - K^^T dX.
// Every exponent is a sum of non-positive log-decays, so nothing overflows for any gate.
//
// One CTA of 512 threads per (b, h).  A forward sweep writes, per chunk, the chunk-start state
// and the chunk's forward quantities (Abar, P, M, X, U) to the workspace; the reverse sweep
// reloads them and applies the lines above, with dS held in shared memory.
#include "common.cuh"
#include "internal.h"

namespace kda {
namespace {

constexpr int BC = 16;     // tokens per chunk
constexpr int BNT = 512;   // threads per CTA
static_assert(2 * BC * BC == BNT, "the dot phase maps a thread pair to each (i, j)");

template <int D>
struct BwdLayout {
    static constexpr int LD = D + 4;              // row stride of states and tiles (floats)
    static constexpr int ST = D * LD;             // one [D][LD] state
    static constexpr int TL = BC * LD;            // one [BC][LD] tile
    static constexpr int CL = BC + 1;             // row stride of the BC x BC matrices
    static constexpr int CC = BC * CL;
    static constexpr int NB = BNT / D;            // row blocks (or value blocks) of threads
    static constexpr int S_ = 0, DS = ST, Q = 2 * ST, K = Q + TL, G = K + TL, V = G + TL, DO = V + TL,
                         U = DO + TL, DU = U + TL, QH = DU + TL, KH = QH + TL, KT = KH + TL;
    static constexpr int AB = KT + TL, P = AB + CC, M = P + CC, DP = M + CC, DA = DP + CC;
    static constexpr int BETA = DA + CC, DBETA = BETA + BC, GC = DBETA + BC, REDK = GC + D, REDS = REDK + NB * D;
    static constexpr int FLOATS = REDS + NB * D;
    static constexpr size_t BYTES = sizeof(float) * FLOATS;
};

__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t u)
{
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}

struct BwdArgs {
    const void *q, *k, *v, *g, *beta;   // io dtype
    const float *s0;                    // [B, H, D, D] or null
    const void *dO;                     // io dtype
    const float *dST;                   // [B, H, D, D] or null
    void *dq, *dk, *dv, *dg, *dbeta;    // io dtype
    float *ds0;                         // [B, H, D, D] or null
    float *ckpt;                        // [B, H, nchunks, ChunkRecord<D>::FLOATS]
    int T, H;
};

// What the forward sweep keeps of each chunk (fp32): the chunk-start state [D][D], U and X =
// V - K^ S [BC][D], then M, P and Abar [BC][BC] (dense).
template <int D>
struct ChunkRecord {
    static constexpr int S = 0, U = D * D, X = U + BC * D, M = X + BC * D, P = M + BC * BC, AB = P + BC * BC;
    static constexpr int FLOATS = AB + BC * BC;
};

template <typename IO, int D>
__global__ void __launch_bounds__(BNT, 1)
kda_backward_kernel(BwdArgs a)
{
    using L = BwdLayout<D>;
    constexpr int LD = L::LD, NB = L::NB, RPT = BC / NB, JPT = D / NB, CL = L::CL;
    extern __shared__ __align__(16) float bsm[];
    float *Ss = bsm + L::S_, *dSs = bsm + L::DS, *Qs = bsm + L::Q, *Ks = bsm + L::K, *Gs = bsm + L::G;
    float *Vs = bsm + L::V, *dOs = bsm + L::DO, *Us = bsm + L::U, *dUs = bsm + L::DU;
    float *QHs = bsm + L::QH, *KHs = bsm + L::KH, *KTs = bsm + L::KT;
    float *ABs = bsm + L::AB, *Ps = bsm + L::P, *Ms = bsm + L::M, *dPs = bsm + L::DP, *dAs = bsm + L::DA;
    float *BETA = bsm + L::BETA, *DBETA = bsm + L::DBETA, *GCs = bsm + L::GC;
    float *REDK = bsm + L::REDK, *REDS = bsm + L::REDS;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x, b = bh / a.H, h = bh % a.H;
    const int T = a.T, H = a.H;
    const int nch = (T + BC - 1) / BC;
    using R = ChunkRecord<D>;
    float *ck = a.ckpt + (size_t)bh * nch * R::FLOATS;
    const size_t soff = (size_t)bh * D * D;
    const int col = tid % D, rb = tid / D;   // column and row block (or value block) of this thread
    auto gidx = [&](int t, int c) -> size_t { return ((size_t)(b * T + t) * H + h) * D + c; };

    // ---------------------------------------------------------------- helpers
    // A chunk's tiles (and, when given, a state) in 16-byte pieces: every thread issues all of
    // its loads before it stores any, so the chunk pays one memory latency, not one per piece.
    constexpr int EPC = 16 / (int)sizeof(IO);          // elements per 16-byte piece
    constexpr int PPT = BC * D / EPC;                  // pieces per tile
    // the tile pointers are chosen by a compare chain, so they stay in registers
    auto pick = [](auto const *arr, int n, int tl) {
        auto r = arr[0];
#pragma unroll
        for (int x = 1; x < 5; ++x)
            if (x < n && tl == x) r = arr[x];
        return r;
    };
    auto load_chunk = [&](float *const *dst, const void *const *src, int ntiles, int t0, float *sdst,
                          const float *ssrc) {
        constexpr int MAXP = (5 * PPT + BNT - 1) / BNT;
        constexpr int SP = D * D / 4 / BNT;            // state float4s per thread
        uint4 raw[MAXP];
        float4 st[SP];
        if (sdst) {
#pragma unroll
            for (int e = 0; e < SP; ++e) {
                const int idx = tid + BNT * e, c = idx / (D / 4), j4 = (idx % (D / 4)) * 4;
                st[e] = ssrc ? *(const float4 *)(ssrc + (size_t)c * D + j4) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
#pragma unroll
        for (int e = 0; e < MAXP; ++e) {
            const int f = tid + BNT * e, tl = f / PPT, pc = f % PPT;
            const int i = pc / (D / EPC), c = (pc % (D / EPC)) * EPC;
            raw[e] = make_uint4(0u, 0u, 0u, 0u);
            if (tl < ntiles && t0 + i < T) raw[e] = *(const uint4 *)((const IO *)pick(src, ntiles, tl) + gidx(t0 + i, c));
        }
        if (sdst) {
#pragma unroll
            for (int e = 0; e < SP; ++e) {
                const int idx = tid + BNT * e, c = idx / (D / 4), j4 = (idx % (D / 4)) * 4;
                *(float4 *)(sdst + c * LD + j4) = st[e];
            }
        }
#pragma unroll
        for (int e = 0; e < MAXP; ++e) {
            const int f = tid + BNT * e, tl = f / PPT, pc = f % PPT;
            const int i = pc / (D / EPC), c = (pc % (D / EPC)) * EPC;
            if (tl < ntiles) {
                float *o = pick(dst, ntiles, tl) + i * LD + c;
                if constexpr (sizeof(IO) == 2) {
                    const float2 x0 = bf16x2_to_float2(raw[e].x), x1 = bf16x2_to_float2(raw[e].y);
                    const float2 x2 = bf16x2_to_float2(raw[e].z), x3 = bf16x2_to_float2(raw[e].w);
                    *(float4 *)o = make_float4(x0.x, x0.y, x1.x, x1.y);
                    *(float4 *)(o + 4) = make_float4(x2.x, x2.y, x3.x, x3.y);
                } else {
                    *(float4 *)o = make_float4(__uint_as_float(raw[e].x), __uint_as_float(raw[e].y),
                                               __uint_as_float(raw[e].z), __uint_as_float(raw[e].w));
                }
            }
        }
    };
    auto load_state = [&](float *dst, const float *src) {
        for (int idx = tid; idx < D * D / 4; idx += BNT) {
            const int c = idx / (D / 4), j4 = (idx % (D / 4)) * 4;
            const float4 x = src ? *(const float4 *)(src + (size_t)c * D + j4) : make_float4(0.f, 0.f, 0.f, 0.f);
            *(float4 *)(dst + c * LD + j4) = x;
        }
    };
    auto store_state = [&](float *dst, const float *src) {
        for (int idx = tid; idx < D * D / 4; idx += BNT) {
            const int c = idx / (D / 4), j4 = (idx % (D / 4)) * 4;
            *(float4 *)(dst + (size_t)c * D + j4) = *(const float4 *)(src + c * LD + j4);
        }
    };
    // G = inclusive cumsum of g over the chunk (in place), G_C, and the decayed q / k tiles
    auto gates = [&](bool with_q) {
        if (tid < D) {
            float acc = 0.0f;
#pragma unroll
            for (int i = 0; i < BC; ++i) {
                acc += Gs[i * LD + tid];
                Gs[i * LD + tid] = acc;
            }
            GCs[tid] = acc;
        }
        __syncthreads();
        for (int idx = tid; idx < BC * D; idx += BNT) {
            const int i = idx / D, c = idx % D;
            const float G = Gs[i * LD + c], kv = Ks[i * LD + c];
            const float e = __expf(G);
            KHs[i * LD + c] = kv * e;
            KTs[i * LD + c] = kv * __expf(GCs[c] - G);
            if (with_q) QHs[i * LD + c] = Qs[i * LD + c] * e;
        }
    };
    // P (j <= i) and Abar (j < i).  Warp w takes the pairs p = w + 16 k (k < 9) of the 136
    // (i, j <= i), lanes over channels; the 9 + 9 per-lane partial sums are then reduced in one
    // transposed butterfly (31 shuffles instead of 18 x 5), after which lane l holds the total
    // of partial l: P of pair k in lane k, Abar of pair k in lane 16 + k.  The pairing of the
    // butterfly is warp_sum's, so the sums are the same to the bit.
    auto pair_dots = [&]() {
        constexpr int NP = BC * (BC + 1) / 2, KP = (NP + 15) / 16;
        static_assert(KP <= 16 && BNT / 32 == 16, "pair mapping");
        float v[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0.0f;
#pragma unroll
        for (int k = 0; k < KP; ++k) {
            const int p = warp + 16 * k;
            if (p < NP) {
                int i = (int)((sqrtf(8.0f * p + 1.0f) - 1.0f) * 0.5f);
                if ((i + 1) * (i + 2) / 2 <= p) ++i;
                if (i * (i + 1) / 2 > p) --i;
                const int j = p - i * (i + 1) / 2;
                float pv = 0.0f, av = 0.0f;
#pragma unroll
                for (int e = 0; e < D / 32; ++e) {
                    const int c = lane + 32 * e;
                    const float x = Ks[j * LD + c] * __expf(Gs[i * LD + c] - Gs[j * LD + c]);
                    pv += Qs[i * LD + c] * x;
                    av += Ks[i * LD + c] * x;
                }
                v[k] = pv;
                v[16 + k] = av;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const bool up = (lane & o) != 0;
#pragma unroll
            for (int e = 0; e < o; ++e) {
                const float keep = up ? v[e + o] : v[e], send = up ? v[e] : v[e + o];
                v[e] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
        }
        const int k = lane & 15, p = warp + 16 * k;
        if (k < KP && p < NP) {
            int i = (int)((sqrtf(8.0f * p + 1.0f) - 1.0f) * 0.5f);
            if ((i + 1) * (i + 2) / 2 <= p) ++i;
            if (i * (i + 1) / 2 > p) --i;
            const int j = p - i * (i + 1) / 2;
            if (lane < 16) Ps[i * CL + j] = v[0];
            else if (j < i) ABs[i * CL + j] = v[0];
        }
    };
    // M = (I + Diag(beta) Abar)^-1 by forward substitution; lane j owns column j (warp 0)
    auto invert = [&]() {
        if (lane < BC) {
            const int j = lane;
            float m[BC];
#pragma unroll
            for (int i = 0; i < BC; ++i) {
                float s = 0.0f;
#pragma unroll
                for (int r = 0; r < i; ++r)
                    if (r >= j) s += ABs[i * CL + r] * m[r];
                m[i] = i < j ? 0.0f : (i == j ? 1.0f : -BETA[i] * s);
            }
#pragma unroll
            for (int i = 0; i < BC; ++i) Ms[i * CL + j] = m[i];
        }
    };
    // X = V - K^ S in place in Vs; (row block, column) partition
    auto ks_x = [&]() {
        float acc[RPT];
#pragma unroll
        for (int r = 0; r < RPT; ++r) acc[r] = 0.0f;
        for (int c = 0; c < D; c += 4) {
            const float s0 = Ss[(c + 0) * LD + col], s1 = Ss[(c + 1) * LD + col];
            const float s2 = Ss[(c + 2) * LD + col], s3 = Ss[(c + 3) * LD + col];
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const float4 kh = *(const float4 *)(KHs + (rb * RPT + r) * LD + c);
                acc[r] += kh.x * s0 + kh.y * s1 + kh.z * s2 + kh.w * s3;
            }
        }
#pragma unroll
        for (int r = 0; r < RPT; ++r) Vs[(rb * RPT + r) * LD + col] -= acc[r];
    };
    // U = M (beta X)
    auto u_from_x = [&]() {
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            const int i = rb * RPT + r;
            float acc = 0.0f;
            for (int m = 0; m <= i; ++m) acc += Ms[i * CL + m] * BETA[m] * Vs[m * LD + col];
            Us[i * LD + col] = acc;
        }
    };

    // ---------------------------------------------------------------- forward sweep: checkpoints
    load_state(Ss, a.s0 ? a.s0 + soff : nullptr);
    __syncthreads();
    for (int n = 0; n < nch; ++n) {
        const int t0 = n * BC;
        float *rec = ck + (size_t)n * R::FLOATS;
        store_state(rec + R::S, Ss);
        {
            float *const dst[4] = {Qs, Ks, Gs, Vs};
            const void *const src[4] = {a.q, a.k, a.g, a.v};
            load_chunk(dst, src, 4, t0, nullptr, nullptr);
        }
        if (tid < BC) BETA[tid] = t0 + tid < T ? to_f32(((const IO *)a.beta)[(size_t)(b * T + t0 + tid) * H + h]) : 0.0f;
        __syncthreads();
        gates(false);
        pair_dots();
        __syncthreads();
        if (warp == 0) invert();
        ks_x();
        __syncthreads();
        u_from_x();
        __syncthreads();
        // the chunk's record for the reverse sweep: U, X (in Vs), M, P, Abar
        for (int idx = tid; idx < BC * D / 4; idx += BNT) {
            const int i = idx / (D / 4), c4 = (idx % (D / 4)) * 4;
            *(float4 *)(rec + R::U + i * D + c4) = *(const float4 *)(Us + i * LD + c4);
            *(float4 *)(rec + R::X + i * D + c4) = *(const float4 *)(Vs + i * LD + c4);
        }
        if (tid < BC * BC) {
            const int i = tid / BC, j = tid % BC;
            rec[R::M + tid] = Ms[i * CL + j];
            rec[R::P + tid] = j <= i ? Ps[i * CL + j] : 0.0f;
            rec[R::AB + tid] = j < i ? ABs[i * CL + j] : 0.0f;
        }
        // S <- Diag(exp G_C) S + K~^T U; (column, value block) partition
        {
            const float gc = __expf(GCs[col]);
            float acc[JPT];
#pragma unroll
            for (int jj = 0; jj < JPT; jj += 4) {
                const float4 x = *(const float4 *)(Ss + col * LD + rb * JPT + jj);
                acc[jj] = gc * x.x; acc[jj + 1] = gc * x.y; acc[jj + 2] = gc * x.z; acc[jj + 3] = gc * x.w;
            }
            for (int i = 0; i < BC; ++i) {
                const float kt = KTs[i * LD + col];
#pragma unroll
                for (int jj = 0; jj < JPT; jj += 4) {
                    const float4 u = *(const float4 *)(Us + i * LD + rb * JPT + jj);
                    acc[jj] += kt * u.x; acc[jj + 1] += kt * u.y; acc[jj + 2] += kt * u.z; acc[jj + 3] += kt * u.w;
                }
            }
#pragma unroll
            for (int jj = 0; jj < JPT; jj += 4)
                *(float4 *)(Ss + col * LD + rb * JPT + jj) = make_float4(acc[jj], acc[jj + 1], acc[jj + 2], acc[jj + 3]);
        }
        __syncthreads();
    }

    // ---------------------------------------------------------------- reverse sweep
    load_state(dSs, a.dST ? a.dST + soff : nullptr);
    for (int n = nch - 1; n >= 0; --n) {
        const int t0 = n * BC;
        const float *rec = ck + (size_t)n * R::FLOATS;
        {
            // the record's U, X, M, P, Abar: loads issued before the chunk's, stored after
            constexpr int NF4 = BC * D / 4, UX = (NF4 + BNT - 1) / BNT;   // float4s of U (of X) per thread
            static_assert(BC * BC <= BNT, "record load mapping");
            float4 ru[UX], rx[UX];
#pragma unroll
            for (int e = 0; e < UX; ++e) {
                const int idx = tid + BNT * e, i = idx / (D / 4), c4 = (idx % (D / 4)) * 4;
                if (idx < NF4) {
                    ru[e] = *(const float4 *)(rec + R::U + i * D + c4);
                    rx[e] = *(const float4 *)(rec + R::X + i * D + c4);
                }
            }
            float rm = 0.0f, rp = 0.0f, ra = 0.0f;
            if (tid < BC * BC) {
                rm = rec[R::M + tid];
                rp = rec[R::P + tid];
                ra = rec[R::AB + tid];
            }
            float *const dst[4] = {Qs, Ks, Gs, dOs};
            const void *const src[4] = {a.q, a.k, a.g, a.dO};
            load_chunk(dst, src, 4, t0, Ss, rec + R::S);
#pragma unroll
            for (int e = 0; e < UX; ++e) {
                const int idx = tid + BNT * e, i = idx / (D / 4), c4 = (idx % (D / 4)) * 4;
                if (idx < NF4) {
                    *(float4 *)(Us + i * LD + c4) = ru[e];
                    *(float4 *)(Vs + i * LD + c4) = rx[e];   // X
                }
            }
            if (tid < BC * BC) {
                const int i = tid / BC, j = tid % BC;
                Ms[i * CL + j] = rm;
                Ps[i * CL + j] = rp;
                ABs[i * CL + j] = ra;
            }
        }
        if (tid < BC) BETA[tid] = t0 + tid < T ? to_f32(((const IO *)a.beta)[(size_t)(b * T + t0 + tid) * H + h]) : 0.0f;
        __syncthreads();
        gates(true);
        __syncthreads();

        // dU = P^T dO + K~ dS_next, (row block, column) partition; then per (row, channel):
        // dq <- exp(G) dO S^T, dk- <- exp(G_C - G) U dS_next^T and its share of dG_C
        float dq[RPT], dkp[RPT], dkm[RPT];
        {
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const int m = rb * RPT + r;
                float acc = 0.0f;
                for (int i = m; i < BC; ++i) acc += Ps[i * CL + m] * dOs[i * LD + col];
                dUs[m * LD + col] = acc;
            }
            float acc[RPT];
#pragma unroll
            for (int r = 0; r < RPT; ++r) acc[r] = 0.0f;
            for (int c = 0; c < D; c += 4) {
                const float s0 = dSs[(c + 0) * LD + col], s1 = dSs[(c + 1) * LD + col];
                const float s2 = dSs[(c + 2) * LD + col], s3 = dSs[(c + 3) * LD + col];
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    const float4 kt = *(const float4 *)(KTs + (rb * RPT + r) * LD + c);
                    acc[r] += kt.x * s0 + kt.y * s1 + kt.z * s2 + kt.w * s3;
                }
            }
#pragma unroll
            for (int r = 0; r < RPT; ++r) dUs[(rb * RPT + r) * LD + col] += acc[r];
        }
        {
            const int c = col;
            float aq[RPT], aw[RPT];
#pragma unroll
            for (int r = 0; r < RPT; ++r) aq[r] = aw[r] = 0.0f;
            for (int j = 0; j < D; j += 4) {
                const float4 s = *(const float4 *)(Ss + c * LD + j);
                const float4 ds = *(const float4 *)(dSs + c * LD + j);
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    const int i = rb * RPT + r;
                    const float4 o = *(const float4 *)(dOs + i * LD + j);
                    const float4 u = *(const float4 *)(Us + i * LD + j);
                    aq[r] += o.x * s.x + o.y * s.y + o.z * s.z + o.w * s.w;
                    aw[r] += u.x * ds.x + u.y * ds.y + u.z * ds.z + u.w * ds.w;
                }
            }
            float kpart = 0.0f;
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const int i = rb * RPT + r;
                const float G = Gs[i * LD + c];
                dq[r] = __expf(G) * aq[r];
                dkm[r] = __expf(GCs[c] - G) * aw[r];
                kpart += Ks[i * LD + c] * dkm[r];
            }
            REDK[rb * D + c] = kpart;
        }
        __syncthreads();
        // dZ = M^T dU, into the K~ tile (free now)
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            const int m = rb * RPT + r;
            float acc = 0.0f;
            for (int i = m; i < BC; ++i) acc += Ms[i * CL + m] * dUs[i * LD + col];
            KTs[m * LD + col] = acc;
        }
        __syncthreads();
        // dP (j <= i), dA (j < i) and rowsum(dZ . X): a thread pair per (i, j), each thread
        // summing one half of the columns
        {
            const int o = tid >> 1, hf = tid & 1, i = o / BC, j = o % BC;
            const float *xo = dOs + i * LD + hf * (D / 2), *xz = KTs + i * LD + hf * (D / 2);
            const float *yu = Us + j * LD + hf * (D / 2), *yx = Vs + i * LD + hf * (D / 2);
            float sp = 0.0f, sa = 0.0f, sb = 0.0f;
#pragma unroll 4
            for (int c = 0; c < D / 2; c += 4) {
                const float4 u = *(const float4 *)(yu + c), x = *(const float4 *)(xo + c);
                const float4 z = *(const float4 *)(xz + c);
                sp += x.x * u.x + x.y * u.y + x.z * u.z + x.w * u.w;
                sa += z.x * u.x + z.y * u.y + z.z * u.z + z.w * u.w;
                if (i == j) {
                    const float4 v = *(const float4 *)(yx + c);
                    sb += z.x * v.x + z.y * v.y + z.z * v.z + z.w * v.w;
                }
            }
            sp += __shfl_xor_sync(0xffffffffu, sp, 1);
            sa += __shfl_xor_sync(0xffffffffu, sa, 1);
            sb += __shfl_xor_sync(0xffffffffu, sb, 1);
            if (hf == 0) {
                if (j <= i) dPs[i * CL + j] = sp;
                if (j < i) dAs[i * CL + j] = -sa;
                if (i == j) DBETA[i] = sb;
            }
        }
        __syncthreads();
        // dbeta += rowsum(dA . Abar), dAbar = Diag(beta) dA (warp 0, lane = row);
        // dX = Diag(beta) dZ in place (everyone)
        if (warp == 0 && lane < BC) {
            const int i = lane;
            float s = 0.0f;
            for (int j = 0; j < i; ++j) {
                const float d = dAs[i * CL + j];
                s += d * ABs[i * CL + j];
                dAs[i * CL + j] = BETA[i] * d;
            }
            DBETA[i] += s;
        }
        for (int idx = tid; idx < BC * D; idx += BNT) {
            const int i = idx / D, c = idx % D;
            KTs[i * LD + c] *= BETA[i];
        }
        __syncthreads();
        // per (row, channel): dk+ <- -exp(G) dX S^T, the pairwise terms, dG; then per
        // (channel, value block): dS <- Diag(exp G_C) dS + Q^^T dO - K^^T dX and the decay
        // share of dG_C
        {
            const int c = col;
            float ax[RPT];
#pragma unroll
            for (int r = 0; r < RPT; ++r) ax[r] = 0.0f;
            for (int j = 0; j < D; j += 4) {
                const float4 s = *(const float4 *)(Ss + c * LD + j);
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    const float4 x = *(const float4 *)(KTs + (rb * RPT + r) * LD + j);
                    ax[r] += x.x * s.x + x.y * s.y + x.z * s.z + x.w * s.w;
                }
            }
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const int i = rb * RPT + r;
                const float Gi = Gs[i * LD + c], qi = Qs[i * LD + c], ki = Ks[i * LD + c];
                float aq = dq[r], ap = -__expf(Gi) * ax[r], am = dkm[r];
                for (int j = 0; j <= i; ++j) {
                    const float e = __expf(Gi - Gs[j * LD + c]) * Ks[j * LD + c];
                    aq += dPs[i * CL + j] * e;
                    if (j < i) ap += dAs[i * CL + j] * e;
                }
                for (int m = i; m < BC; ++m) {
                    const float e = __expf(Gs[m * LD + c] - Gi);
                    float w = dPs[m * CL + i] * Qs[m * LD + c];
                    if (m > i) w += dAs[m * CL + i] * Ks[m * LD + c];
                    am += w * e;
                }
                dq[r] = aq;
                dkp[r] = ap;
                dkm[r] = am;
                dUs[i * LD + c] = qi * aq + ki * ap - ki * am;   // dG (dU is consumed)
                if (t0 + i < T) {
                    ((IO *)a.dq)[gidx(t0 + i, c)] = from_f32<IO>(aq);
                    ((IO *)a.dk)[gidx(t0 + i, c)] = from_f32<IO>(ap + am);
                }
            }
        }
        {
            const float gc = __expf(GCs[col]);
            float acc[JPT];
            float dec = 0.0f;
#pragma unroll
            for (int jj = 0; jj < JPT; jj += 4) {
                const float4 ds = *(const float4 *)(dSs + col * LD + rb * JPT + jj);
                const float4 sv = *(const float4 *)(Ss + col * LD + rb * JPT + jj);
                dec += ds.x * sv.x + ds.y * sv.y + ds.z * sv.z + ds.w * sv.w;
                acc[jj] = gc * ds.x; acc[jj + 1] = gc * ds.y; acc[jj + 2] = gc * ds.z; acc[jj + 3] = gc * ds.w;
            }
            REDS[rb * D + col] = gc * dec;
            for (int i = 0; i < BC; ++i) {
                const float qh = QHs[i * LD + col], kh = KHs[i * LD + col];
#pragma unroll
                for (int jj = 0; jj < JPT; jj += 4) {
                    const float4 o = *(const float4 *)(dOs + i * LD + rb * JPT + jj);
                    const float4 x = *(const float4 *)(KTs + i * LD + rb * JPT + jj);
                    acc[jj] += qh * o.x - kh * x.x; acc[jj + 1] += qh * o.y - kh * x.y;
                    acc[jj + 2] += qh * o.z - kh * x.z; acc[jj + 3] += qh * o.w - kh * x.w;
                }
            }
#pragma unroll
            for (int jj = 0; jj < JPT; jj += 4)
                *(float4 *)(dSs + col * LD + rb * JPT + jj) = make_float4(acc[jj], acc[jj + 1], acc[jj + 2], acc[jj + 3]);
        }
        __syncthreads();
        // dg = reverse cumsum of dG, with dG_C added to the last row; dv = dX; dbeta
        if (tid < D) {
            float acc = 0.0f;
#pragma unroll
            for (int r = 0; r < NB; ++r) acc += REDK[r * D + tid] + REDS[r * D + tid];
            for (int i = BC - 1; i >= 0; --i) {
                acc += dUs[i * LD + tid];
                if (t0 + i < T) ((IO *)a.dg)[gidx(t0 + i, tid)] = from_f32<IO>(acc);
            }
        }
        for (int idx = tid; idx < BC * D; idx += BNT) {
            const int i = idx / D, c = idx % D;
            if (t0 + i < T) ((IO *)a.dv)[gidx(t0 + i, c)] = from_f32<IO>(KTs[i * LD + c]);
        }
        if (tid < BC && t0 + tid < T) ((IO *)a.dbeta)[(size_t)(b * T + t0 + tid) * H + h] = from_f32<IO>(DBETA[tid]);
        __syncthreads();
    }
    if (a.ds0) store_state(a.ds0 + soff, dSs);
}

template <typename IO, int D>
cudaError_t launch_bwd_t(const BwdArgs &a, int B, cudaStream_t s)
{
    struct Tag;
    const cudaError_t attr = smem_opt_in<Tag>((const void *)kda_backward_kernel<IO, D>, (int)BwdLayout<D>::BYTES);
    if (attr != cudaSuccess) return attr;
    kda_backward_kernel<IO, D><<<B * a.H, BNT, BwdLayout<D>::BYTES, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

size_t backward_workspace_bytes(int B, int T, int H, int d)
{
    const size_t nch = (size_t)(T + BC - 1) / BC;
    const size_t rec = d == 128 ? ChunkRecord<128>::FLOATS : ChunkRecord<64>::FLOATS;
    return (size_t)B * H * nch * rec * sizeof(float);
}

cudaError_t launch_backward(const BackwardArgs &x, cudaStream_t s)
{
    BwdArgs a{x.q, x.k, x.v, x.g, x.beta, x.s0, x.dO, x.dST, x.dq, x.dk, x.dv, x.dg, x.dbeta, x.ds0,
              x.ckpt, x.T, x.H};
    if (x.io == IO_F32) return x.d == 128 ? launch_bwd_t<float, 128>(a, x.B, s) : launch_bwd_t<float, 64>(a, x.B, s);
    return x.d == 128 ? launch_bwd_t<__nv_bfloat16, 128>(a, x.B, s) : launch_bwd_t<__nv_bfloat16, 64>(a, x.B, s);
}

}  // namespace kda
