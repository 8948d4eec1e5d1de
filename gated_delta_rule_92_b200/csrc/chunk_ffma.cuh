// chunk_ffma.cuh -- chunk-parallel GDN-2 forward on CUDA cores (fp32 products).
//
// The recurrence (burn-gdn2 README, "Architecture") regrouped over chunks of
// C = 16, 32 or 64 tokens ("Chunk WY (train)" mode; "Configuration":
// chunk_size, default 64).  For one chunk with
// chunk-start state S (d_k x d_v), per key channel c and local row r:
//     g_r   = sum_{s<=r} log_alpha_s           gamma_r = exp(g_r)
//     Q~_r  = q_r . gamma_r     K~_i = k_i / gamma_i     E_r = b_r . k_r . gamma_r
//     A_ri  = E_r . K~_i  (i < r)      P_ri = Q~_r . K~_i  (i <= r)
//     T     = (I + A)^{-1}             (unit lower triangular)
//     U     = T (W.V) - T (E S)        (the corrected writes u_r)
//     O     = Q~ S + P U
//     S'    = diag(gamma_C) (S + K~^T U)
// which unrolls u_r = w_r.v_r - (diag(alpha_r) S_{r-1})^T (b_r.k_r) over the
// chunk: (I + A) U = W.V - E S.  Every product here is an fp32 FMA, so this
// kernel meets fp32-I/O tolerances; it also cross-checks the tensor-core
// kernel, which evaluates the same products on tcgen05 in a different order.
// 1 / gamma grows with the chunk's decay: a chunk that decays by more than
// e^-kMaxCudaCoreSpan in some channel runs token by token instead
// (chunk_token_steps), which is exact for any decay.
//
// One block of 256 threads per (b, h, 64-column slice of d_v); everything
// for one chunk lives in shared memory (about 215 KB at d_k = 128, C = 64).
#pragma once
#include "decode.cuh"
#include "gdn2_device.cuh"

namespace gdn2 {

// Largest decay of one chunk, in natural-log units (-sum_r log_alpha_r per
// channel), for which the chunked products are evaluated: 1/gamma stays below
// e^60, so neither the products nor the state update can overflow.  A chunk
// past it runs token by token (chunk_token_steps), which is exact for any decay.
constexpr float kMaxCudaCoreSpan = 60.f;

// One chunk of the recurrence token by token on a 256-thread block, from the
// chunk's tiles in shared memory (fp32, the input prep already applied):
//     r_j = sum_c (b_c k_c alpha_c) S_cj,   p_j = sum_c (q_c alpha_c) S_cj,
//     u_j = (w.v)_j - r_j,   S_cj <- alpha_c S_cj + k_c u_j,   o_j = p_j + (q . k) u_j
// with P pseudo-rows per token (GDN-2: P = 1, row t; the second erase
// direction: P = 2, rows 2t (key) and 2t + 1 (query direction, value 0)),
// whose erase reads all see the same decayed state.  Row layouts: q [C][LK]
// per token, kappa and erase vectors (erase already times kappa) [P C][LK],
// alpha [C][LK] (already exp(log_alpha)), values [P C][LV], q . kappa [C][P];
// the state slice S [DK][LV] is read at the start and written back at the end.
// Thread (j, part): value column j = tid / 4, rows part, part + 4, ... of it.
template <int DK, int NV, int P, typename IO>
__device__ __forceinline__ void chunk_token_steps(const float *sQ, const float *sKap, const float *sEr,
                                                  const float *sAl, const float *sVal, const float *sQK,
                                                  float *sS, int LK, int LV, int rows, IO *__restrict__ o,
                                                  long o_row0, long o_stride) {
    static_assert(NV == 64, "one column per four threads");
    constexpr int RPT = DK / 4;
    const int tid = threadIdx.x, j = tid >> 2, part = tid & 3;
    float Sr[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i) Sr[i] = sS[(4 * i + part) * LV + j];
    for (int t = 0; t < rows; ++t) {
        float rr[P], pq = 0.f;
#pragma unroll
        for (int x = 0; x < P; ++x) rr[x] = 0.f;
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const int c = 4 * i + part;
            const float a = sAl[t * LK + c], sa = a * Sr[i];
            pq = fmaf(sQ[t * LK + c], sa, pq);
#pragma unroll
            for (int x = 0; x < P; ++x) rr[x] = fmaf(sEr[(P * t + x) * LK + c], sa, rr[x]);
        }
#pragma unroll
        for (int off = 1; off < 4; off <<= 1) {
            pq += __shfl_xor_sync(0xffffffffu, pq, off);
#pragma unroll
            for (int x = 0; x < P; ++x) rr[x] += __shfl_xor_sync(0xffffffffu, rr[x], off);
        }
        float u[P], ov = pq;
#pragma unroll
        for (int x = 0; x < P; ++x) {
            u[x] = sVal[(P * t + x) * LV + j] - rr[x];
            ov = fmaf(sQK[P * t + x], u[x], ov);
        }
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const int c = 4 * i + part;
            float nv = sAl[t * LK + c] * Sr[i];
#pragma unroll
            for (int x = 0; x < P; ++x) nv = fmaf(sKap[(P * t + x) * LK + c], u[x], nv);
            Sr[i] = nv;
        }
        IO *dst = o + o_row0 + (long)t * o_stride + j;
        if (part == 0 && GDN2_IN_BOUNDS(kBufO, dst, sizeof(IO))) {
            if constexpr (sizeof(IO) == 4) *dst = ov;
            else *dst = __float2bfloat16_rn(ov);
        }
    }
#pragma unroll
    for (int i = 0; i < RPT; ++i) sS[(4 * i + part) * LV + j] = Sr[i];
}

template <int DK, int CH = 64>
struct FfmaCfg {
    static_assert(CH == 16 || CH == 32 || CH == 64, "chunk length");
    static constexpr int C = CH;
    static constexpr int NV = 64;
    static constexpr int LK = DK + 1;   // padded row stride for [C][DK] tiles
    static constexpr int LC = C + 1;    // padded row stride for [C][C] tiles (A, P, T)
    static constexpr int LV = NV + 1;   // padded row stride for [.][NV] tiles (W.V, U, S)
    // float offsets
    static constexpr int O_Q = 0;
    static constexpr int O_K = O_Q + C * LK;
    static constexpr int O_E = O_K + C * LK;
    static constexpr int O_G = O_E + C * LK;            // log-decay, then A and P
    static constexpr int G_SIZE = (C * LK > 2 * C * LC) ? C * LK : 2 * C * LC;
    static constexpr int O_T = O_G + G_SIZE;
    static constexpr int O_WV = O_T + C * LC;           // W.V, then E S
    static constexpr int O_U = O_WV + C * LV;           // T (W.V), then U
    static constexpr int O_S = O_U + C * LV;            // state slice [DK][NV]
    static constexpr int O_GC = O_S + DK * LV;
    static constexpr int FLOATS = O_GC + DK;
    static constexpr size_t BYTES = sizeof(float) * FLOATS;
};

// FUSED with fz.prep reads raw q, k, b, w: rows of q and k are L2-normalised
// over d_k (x / sqrt(sum x^2 + l2_eps)), b = sigmoid(b) (x2 with neg_eigval),
// w = sigmoid(w).  The output epilogue of this path runs as a separate pass.
template <typename IO, int DK, bool FUSED = false, int CH = 64>
__global__ void __launch_bounds__(256, 1)
chunk_fwd_ffma_kernel(const IO *__restrict__ q, const IO *__restrict__ k, const IO *__restrict__ v,
                      const IO *__restrict__ la, const IO *__restrict__ bg, const IO *__restrict__ wg,
                      const float *__restrict__ S0, IO *__restrict__ o, float *__restrict__ S_T,
                      int T, int H, int HV, int d_v, const int *__restrict__ cu_seqlens,
                      const FuseArgs fz = {}) {
    const bool prep = FUSED && fz.prep;
    const float bscale = (FUSED && fz.neg_eigval) ? 2.f : 1.f;
    using Cfg = FfmaCfg<DK, CH>;
    constexpr int C = Cfg::C, NV = Cfg::NV, LK = Cfg::LK, LC = Cfg::LC, LV = Cfg::LV;
    extern __shared__ float sm[];
    float *sQ = sm + Cfg::O_Q, *sK = sm + Cfg::O_K, *sE = sm + Cfg::O_E, *sG = sm + Cfg::O_G;
    float *sA = sG, *sP = sG + C * LC;
    float *sT = sm + Cfg::O_T, *sWV = sm + Cfg::O_WV, *sU = sm + Cfg::O_U, *sS = sm + Cfg::O_S;
    float *sGC = sm + Cfg::O_GC;

    const int tid = threadIdx.x;
    // value head hv (of HV) reads key head h = hv / (HV / H); sequence bb is
    // tokens [tok_base, tok_base + len): bb * T + [0, T), or [cu[bb], cu[bb+1])
    const int j0 = blockIdx.x * NV, hv = blockIdx.y, bb = blockIdx.z;
    const int h = hv / (HV / H);
    long tok_base = (long)bb * T;
    int len = T;
    if (cu_seqlens != nullptr) {
        const int a = GDN2_IN_BOUNDS(kBufCU, cu_seqlens + bb, sizeof(int)) ? cu_seqlens[bb] : -1;
        const int e = GDN2_IN_BOUNDS(kBufCU, cu_seqlens + bb + 1, sizeof(int)) ? cu_seqlens[bb + 1] : -1;
        if (a < 0 || e < a || e > T) {   // malformed packing: this sequence is skipped
            if (threadIdx.x == 0) record_status(kStatusBadArgs);
            return;
        }
        tok_base = a;
        len = e - a;
    }
    const long head = (long)bb * HV + hv;
    const int NC = (len + C - 1) / C;   // the last chunk may be partial (padded rows are zeros)

    // initial state slice
    for (int idx = tid; idx < DK * NV; idx += 256) {
        const int c = idx / NV, j = idx % NV;
        const float *sp = S0 ? S0 + (head * DK + c) * d_v + j0 + j : nullptr;
        sS[c * LV + j] = (sp && GDN2_IN_BOUNDS(kBufS0, sp, 4)) ? *sp : 0.f;
    }

    for (int n = 0; n < NC; ++n) {
        const long tok0 = tok_base + (long)n * C;   // token row of local r = 0
        const int rows = min(C, len - n * C);        // valid rows of this chunk
        __syncthreads();
        // ---- load the chunk (fp32 in shared memory); rows past T are zeros,
        // which leaves the recurrence unchanged (k = q = b = w = 0, no decay)
        for (int idx = tid; idx < C * DK; idx += 256) {
            const int r = idx / DK, c = idx % DK;
            const long g = ((tok0 + r) * H + h) * DK + c;
            const bool in = r < rows;
            sQ[r * LK + c] = (in && GDN2_IN_BOUNDS(kBufQ, q + g, sizeof(IO))) ? ld_io(q + g) : 0.f;
            sK[r * LK + c] = (in && GDN2_IN_BOUNDS(kBufK, k + g, sizeof(IO))) ? ld_io(k + g) : 0.f;
            const float bx = (in && GDN2_IN_BOUNDS(kBufB, bg + g, sizeof(IO))) ? ld_io(bg + g) : 0.f;
            sE[r * LK + c] = in ? (prep ? bscale * sigmoid_f32(bx) : bx) : 0.f;
            sG[r * LK + c] = (in && GDN2_IN_BOUNDS(kBufLA, la + g, sizeof(IO))) ? ld_io(la + g) : 0.f;
        }
        for (int idx = tid; idx < C * NV; idx += 256) {
            const int r = idx / NV, j = idx % NV;
            const long g = ((tok0 + r) * HV + hv) * d_v + j0 + j;
            const bool in = r < rows;
            const float wv = (in && GDN2_IN_BOUNDS(kBufW, wg + g, sizeof(IO))) ? ld_io(wg + g) : 0.f;
            const float vv = (in && GDN2_IN_BOUNDS(kBufV, v + g, sizeof(IO))) ? ld_io(v + g) : 0.f;
            sWV[r * LV + j] = in ? (prep ? sigmoid_f32(wv) : wv) * vv : 0.f;
        }
        __syncthreads();
        if (prep) {   // L2-normalise each row of q and k: warp w takes rows w, w + 8, ...
            const int wp = tid >> 5, l = tid & 31;
            for (int r = wp; r < C; r += 8) {
                float sq = 0.f, sk = 0.f;
                for (int c = l; c < DK; c += 32) {
                    sq = fmaf(sQ[r * LK + c], sQ[r * LK + c], sq);
                    sk = fmaf(sK[r * LK + c], sK[r * LK + c], sk);
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    sq += __shfl_xor_sync(0xffffffffu, sq, off);
                    sk += __shfl_xor_sync(0xffffffffu, sk, off);
                }
                const float iq = l2_inv(sq, fz.l2_eps), ik = l2_inv(sk, fz.l2_eps);
                for (int c = l; c < DK; c += 32) {
                    sQ[r * LK + c] *= iq;
                    sK[r * LK + c] *= ik;
                }
            }
            __syncthreads();
        }
        // ---- the chunk's decay: past kMaxCudaCoreSpan it runs token by token
        {
            float tot = 0.f;
            if (tid < DK)
                for (int r = 0; r < C; ++r) tot += sG[r * LK + tid];
            if (__syncthreads_or(tid < DK && !(tot >= -kMaxCudaCoreSpan))) {
                // erase vectors b.k, alpha = exp(log_alpha) and q . k per token, in place
                for (int idx = tid; idx < C * DK; idx += 256) {
                    const int r = idx / DK, c = idx % DK;
                    sE[r * LK + c] *= sK[r * LK + c];
                    sG[r * LK + c] = __expf(sG[r * LK + c]);
                }
                {
                    const int wp = tid >> 5, l = tid & 31;
                    for (int r = wp; r < C; r += 8) {
                        float qk = 0.f;
                        for (int c = l; c < DK; c += 32) qk = fmaf(sQ[r * LK + c], sK[r * LK + c], qk);
#pragma unroll
                        for (int off = 16; off > 0; off >>= 1) qk += __shfl_xor_sync(0xffffffffu, qk, off);
                        if (l == 0) sGC[r] = qk;
                    }
                }
                __syncthreads();
                chunk_token_steps<DK, NV, 1, IO>(sQ, sK, sE, sG, sWV, sGC, sS, LK, LV, rows, o,
                                                 (tok0 * HV + hv) * (long)d_v + j0, (long)HV * d_v);
                continue;   // the next chunk starts with a barrier
            }
        }
        // ---- cumulative log-decay per key channel and the scaled operands
        if (tid < DK) {
            const int c = tid;
            float g = 0.f;
            for (int r = 0; r < C; ++r) {
                g += sG[r * LK + c];
                const float gam = expf(g), inv = expf(-g);
                const float kv = sK[r * LK + c];
                sQ[r * LK + c] *= gam;
                sE[r * LK + c] = sE[r * LK + c] * kv * gam;
                sK[r * LK + c] = kv * inv;
            }
            sGC[c] = expf(g);
        }
        __syncthreads();
        // ---- A (strictly lower) and P (lower, inclusive); overwrite the log-decay.
        // Register tiles of TC x TC (thread: rows TC (tid / 16).., columns TC (tid % 16)..);
        // a tile wholly above the diagonal is zero without work.
        constexpr int TC = C / 16;
        {
            const int rt = tid >> 4, ct = tid & 15;
            float aa[TC][TC] = {}, pp[TC][TC] = {};
            if (ct <= rt) {
                for (int c = 0; c < DK; ++c) {
                    float e[TC], qq[TC], kk[TC];
#pragma unroll
                    for (int x = 0; x < TC; ++x) {
                        e[x] = sE[(TC * rt + x) * LK + c];
                        qq[x] = sQ[(TC * rt + x) * LK + c];
                        kk[x] = sK[(TC * ct + x) * LK + c];
                    }
#pragma unroll
                    for (int x = 0; x < TC; ++x)
#pragma unroll
                        for (int y = 0; y < TC; ++y) {
                            aa[x][y] = fmaf(e[x], kk[y], aa[x][y]);
                            pp[x][y] = fmaf(qq[x], kk[y], pp[x][y]);
                        }
                }
            }
#pragma unroll
            for (int x = 0; x < TC; ++x)
#pragma unroll
                for (int y = 0; y < TC; ++y) {
                    const int r = TC * rt + x, i = TC * ct + y;
                    sA[r * LC + i] = (i < r) ? aa[x][y] : 0.f;
                    sP[r * LC + i] = (i <= r) ? pp[x][y] : 0.f;
                }
        }
        __syncthreads();
        // ---- T = (I + A)^{-1}: column j by 256 / C threads (rows r = TPC m + qd),
        // right-looking: once row i of the column is final it is broadcast from its
        // owner and every later row takes its term; rows above j stay zero
        {
            constexpr int TPC = 256 / C, RPC = C / TPC;
            const int j = tid / TPC, qd = tid % TPC, lane = tid & 31;
            float acc[RPC];
#pragma unroll
            for (int m = 0; m < RPC; ++m) acc[m] = (TPC * m + qd == j) ? 1.f : 0.f;
#pragma unroll
            for (int i = 0; i < C; ++i) {
                const float xi = __shfl_sync(0xffffffffu, acc[i / TPC], (lane & ~(TPC - 1)) | (i % TPC));
#pragma unroll
                for (int m = i / TPC; m < RPC; ++m) {
                    const int r = TPC * m + qd;
                    if (r > i) acc[m] = fmaf(-sA[r * LC + i], xi, acc[m]);
                }
            }
#pragma unroll
            for (int m = 0; m < RPC; ++m) sT[(TPC * m + qd) * LC + j] = acc[m];
        }
        __syncthreads();
        // ---- U = T (W.V) - T (E S), TC x 4 register tiles of the C x NV result
        {
            const int rt = tid >> 4, ct = tid & 15;
            float u1[TC][4] = {}, es[TC][4] = {};
            for (int i = 0; i < TC * rt + TC; ++i) {   // T is lower triangular
                float tt[TC], vv[4];
#pragma unroll
                for (int x = 0; x < TC; ++x) tt[x] = sT[(TC * rt + x) * LC + i];
#pragma unroll
                for (int y = 0; y < 4; ++y) vv[y] = sWV[i * LV + 4 * ct + y];
#pragma unroll
                for (int x = 0; x < TC; ++x)
#pragma unroll
                    for (int y = 0; y < 4; ++y) u1[x][y] = fmaf(tt[x], vv[y], u1[x][y]);
            }
            for (int c = 0; c < DK; ++c) {
                float e[TC], ss[4];
#pragma unroll
                for (int x = 0; x < TC; ++x) e[x] = sE[(TC * rt + x) * LK + c];
#pragma unroll
                for (int y = 0; y < 4; ++y) ss[y] = sS[c * LV + 4 * ct + y];
#pragma unroll
                for (int x = 0; x < TC; ++x)
#pragma unroll
                    for (int y = 0; y < 4; ++y) es[x][y] = fmaf(e[x], ss[y], es[x][y]);
            }
            __syncthreads();   // everyone has read W.V before E S replaces it
#pragma unroll
            for (int x = 0; x < TC; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) sWV[(TC * rt + x) * LV + 4 * ct + y] = es[x][y];
            __syncthreads();
            for (int i = 0; i < TC * rt + TC; ++i) {
                float tt[TC], vv[4];
#pragma unroll
                for (int x = 0; x < TC; ++x) tt[x] = sT[(TC * rt + x) * LC + i];
#pragma unroll
                for (int y = 0; y < 4; ++y) vv[y] = sWV[i * LV + 4 * ct + y];
#pragma unroll
                for (int x = 0; x < TC; ++x)
#pragma unroll
                    for (int y = 0; y < 4; ++y) u1[x][y] = fmaf(-tt[x], vv[y], u1[x][y]);
            }
#pragma unroll
            for (int x = 0; x < TC; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) sU[(TC * rt + x) * LV + 4 * ct + y] = u1[x][y];
        }
        __syncthreads();
        // ---- O = Q~ S + P U, TC x 4 register tiles
        {
            const int rt = tid >> 4, ct = tid & 15;
            float ov[TC][4] = {};
            for (int c = 0; c < DK; ++c) {
                float qq[TC], ss[4];
#pragma unroll
                for (int x = 0; x < TC; ++x) qq[x] = sQ[(TC * rt + x) * LK + c];
#pragma unroll
                for (int y = 0; y < 4; ++y) ss[y] = sS[c * LV + 4 * ct + y];
#pragma unroll
                for (int x = 0; x < TC; ++x)
#pragma unroll
                    for (int y = 0; y < 4; ++y) ov[x][y] = fmaf(qq[x], ss[y], ov[x][y]);
            }
            for (int i = 0; i < TC * rt + TC; ++i) {   // P is lower triangular
                float pv[TC], uu[4];
#pragma unroll
                for (int x = 0; x < TC; ++x) pv[x] = sP[(TC * rt + x) * LC + i];
#pragma unroll
                for (int y = 0; y < 4; ++y) uu[y] = sU[i * LV + 4 * ct + y];
#pragma unroll
                for (int x = 0; x < TC; ++x)
#pragma unroll
                    for (int y = 0; y < 4; ++y) ov[x][y] = fmaf(pv[x], uu[y], ov[x][y]);
            }
#pragma unroll
            for (int x = 0; x < TC; ++x) {
                const int r = TC * rt + x;
                if (r < rows) {
                    const long g = ((tok0 + r) * HV + hv) * d_v + j0 + 4 * ct;
#pragma unroll
                    for (int y = 0; y < 4; ++y) {
                        if (!GDN2_IN_BOUNDS(kBufO, o + g + y, sizeof(IO))) continue;
                        if constexpr (sizeof(IO) == 4) o[g + y] = ov[x][y];
                        else o[g + y] = __float2bfloat16_rn(ov[x][y]);
                    }
                }
            }
        }
        __syncthreads();
        // ---- S <- diag(gamma_C) (S + K~^T U), 4 x 8 register tiles of the DK x NV state
        for (int tile = tid; tile < (DK / 4) * (NV / 8); tile += 256) {
            const int rt = tile / (NV / 8), ct = tile % (NV / 8);
            float sv[4][8];
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 8; ++y) sv[x][y] = sS[(4 * rt + x) * LV + 8 * ct + y];
            for (int i = 0; i < C; ++i) {
                float kk[4], uu[8];
#pragma unroll
                for (int x = 0; x < 4; ++x) kk[x] = sK[i * LK + 4 * rt + x];
#pragma unroll
                for (int y = 0; y < 8; ++y) uu[y] = sU[i * LV + 8 * ct + y];
#pragma unroll
                for (int x = 0; x < 4; ++x)
#pragma unroll
                    for (int y = 0; y < 8; ++y) sv[x][y] = fmaf(kk[x], uu[y], sv[x][y]);
            }
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const float gcx = sGC[4 * rt + x];
#pragma unroll
                for (int y = 0; y < 8; ++y) sS[(4 * rt + x) * LV + 8 * ct + y] = gcx * sv[x][y];
            }
        }
    }
    __syncthreads();
    if (S_T) {
        for (int idx = tid; idx < DK * NV; idx += 256) {
            const int c = idx / NV, j = idx % NV;
            float *sp = S_T + (head * DK + c) * d_v + j0 + j;
            if (GDN2_IN_BOUNDS(kBufST, sp, 4)) *sp = sS[c * LV + j];
        }
    }
}

}  // namespace gdn2
