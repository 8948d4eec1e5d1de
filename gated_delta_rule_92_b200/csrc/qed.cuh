// qed.cuh -- GDN-2 with the second, query-derived erase direction.
//
// "The Query Knows What to Forget" (mlsanity 2608.13668, abstract): a second
// erase direction, taken from the query and orthogonal to the key, cancels
// what the old state holds along the query.  The page prints no formula; the
// reading built here is
//     r_t = q_t - ((q_t . k_t) / (k_t . k_t)) k_t,   u_t = r_t / sqrt(r_t . r_t + eps)
//     S_t = (I - k_t (b_t . k_t)^T - u_t (c_t . u_t)^T) diag(alpha_t) S_{t-1} + k_t (w_t . v_t)^T
//     o_t = S_t^T q_t
// with c_t a second erase gate on the key axis.  Both erases act on the same
// decayed state, one rank-2 edit per token.  CUDA cores, fp32 products.
#pragma once
#include "chunk_ffma.cuh"
#include "decode.cuh"
#include "gdn2_device.cuh"

namespace gdn2 {

// Sum of `x` over the DK threads 0..DK-1 of the block (the others pass 0):
// warp shuffles, then the DK / 32 warp totals through `scratch` (DK / 32 floats).
// Every thread of the block must call it.
template <int DK>
__device__ __forceinline__ float block_sum_dk(float x, float *scratch) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    if ((threadIdx.x & 31) == 0 && threadIdx.x < DK) scratch[threadIdx.x >> 5] = x;
    __syncthreads();
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < DK / 32; ++w) t += scratch[w];
    __syncthreads();
    return t;
}

// The same for two values at once (one exchange through `scratch`, DK / 32 float2).
template <int DK>
__device__ __forceinline__ float2 block_sum2_dk(float2 x, float2 *scratch) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        x.x += __shfl_xor_sync(0xffffffffu, x.x, off);
        x.y += __shfl_xor_sync(0xffffffffu, x.y, off);
    }
    if ((threadIdx.x & 31) == 0 && threadIdx.x < DK) scratch[threadIdx.x >> 5] = x;
    __syncthreads();
    float2 t = make_float2(0.f, 0.f);
#pragma unroll
    for (int w = 0; w < DK / 32; ++w) {
        t.x += scratch[w].x;
        t.y += scratch[w].y;
    }
    __syncthreads();
    return t;
}

// One decode step per (b, h, NVD-column slice of d_v), 256 threads.  Per
// value column j, with S = S_{t-1} and the decay alpha:
//     r1_j = sum_i (b_i k_i alpha_i) S_ij,  r2_j = sum_i (c_i u_i alpha_i) S_ij,
//     p_j  = sum_i (q_i alpha_i) S_ij,      x_j  = w_j v_j - r1_j
//     S_ij <- alpha_i S_ij + k_i x_j - u_i r2_j
//     o_j  = p_j + (q . k) x_j - (q . u) r2_j,   q . u = |r|^2 / sqrt(|r|^2 + eps)
// S is read once and written once, as in the GDN-2 step.
template <typename IO, int DK, int NVD>
__global__ void __launch_bounds__(256, 2)
decode_step_qed_kernel(const IO *__restrict__ q, const IO *__restrict__ k, const IO *__restrict__ v,
                       const IO *__restrict__ la, const IO *__restrict__ bg, const IO *__restrict__ cg_,
                       const IO *__restrict__ wg, float *__restrict__ S, IO *__restrict__ o, int d_v,
                       float qed_eps) {
    constexpr int TPR = NVD / 4;   // threads across one row of the slice
    constexpr int RG = 256 / TPR;  // thread rows
    constexpr int RPT = DK / RG;   // state rows per thread
    static_assert(RPT >= 1 && RG * RPT == DK, "bad decode tiling");

    __shared__ float s_alpha[DK], s_e1[DK], s_e2[DK], s_qa[DK], s_k[DK], s_u[DK];
    __shared__ float s_wv[NVD];
    __shared__ __align__(16) float s_red[3][RG][NVD];
    __shared__ float s_scr[DK / 32];
    __shared__ float2 s_scr2[DK / 32];

    const int tid = threadIdx.x;
    const int cgr = tid % TPR;   // float4 column group
    const int rg = tid / TPR;    // thread row
    const long bh = blockIdx.x;
    const int j0 = blockIdx.y * NVD;

    float *Sh = S + bh * (long)DK * d_v + j0 + cgr * 4;
    float4 s[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const float4 *sp = reinterpret_cast<const float4 *>(Sh + (long)(i * RG + rg) * d_v);
        s[i] = GDN2_IN_BOUNDS(kBufS0, sp, 16) ? __ldcs(sp) : make_float4(0.f, 0.f, 0.f, 0.f);
    }

    float qv = 0.f, kv = 0.f, bv = 0.f, cv = 0.f, lv = 0.f;
    if (tid < DK) {
        const long off = bh * DK + tid;
        qv = GDN2_IN_BOUNDS(kBufQ, q + off, sizeof(IO)) ? ld_io(q + off) : 0.f;
        kv = GDN2_IN_BOUNDS(kBufK, k + off, sizeof(IO)) ? ld_io(k + off) : 0.f;
        bv = GDN2_IN_BOUNDS(kBufB, bg + off, sizeof(IO)) ? ld_io(bg + off) : 0.f;
        cv = GDN2_IN_BOUNDS(kBufC, cg_ + off, sizeof(IO)) ? ld_io(cg_ + off) : 0.f;
        lv = GDN2_IN_BOUNDS(kBufLA, la + off, sizeof(IO)) ? ld_io(la + off) : 0.f;
    }
    // the query's part orthogonal to the key, normalised
    const float2 qkk = block_sum2_dk<DK>(make_float2(qv * kv, kv * kv), s_scr2);
    const float qk = qkk.x, kk = qkk.y;
    const float coef = kk > 0.f ? qk / kk : 0.f;
    const float rv = qv - coef * kv;
    const float rr = block_sum_dk<DK>(rv * rv, s_scr);
    const float den = rr + qed_eps;
    const float nu = den > 0.f ? rsqrtf(den) : 0.f;
    const float qu = rr * nu;   // q . u = r . r / sqrt(r . r + eps)
    if (tid < DK) {
        const float a = __expf(lv), uv = rv * nu;
        s_alpha[tid] = a;
        s_e1[tid] = bv * kv * a;
        s_e2[tid] = cv * uv * a;
        s_qa[tid] = qv * a;
        s_k[tid] = kv;
        s_u[tid] = uv;
    }
    if (tid < NVD) {
        const long vo = bh * (long)d_v + j0 + tid;
        s_wv[tid] = (GDN2_IN_BOUNDS(kBufW, wg + vo, sizeof(IO)) ? ld_io(wg + vo) : 0.f) *
                    (GDN2_IN_BOUNDS(kBufV, v + vo, sizeof(IO)) ? ld_io(v + vo) : 0.f);
    }
    __syncthreads();

    // partial column sums over this thread's rows
    float4 a1 = make_float4(0.f, 0.f, 0.f, 0.f), a2 = a1, ap = a1;
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int row = i * RG + rg;
        const float e1 = s_e1[row], e2 = s_e2[row], qa = s_qa[row];
        a1.x += e1 * s[i].x; a1.y += e1 * s[i].y; a1.z += e1 * s[i].z; a1.w += e1 * s[i].w;
        a2.x += e2 * s[i].x; a2.y += e2 * s[i].y; a2.z += e2 * s[i].z; a2.w += e2 * s[i].w;
        ap.x += qa * s[i].x; ap.y += qa * s[i].y; ap.z += qa * s[i].z; ap.w += qa * s[i].w;
    }
    *reinterpret_cast<float4 *>(&s_red[0][rg][cgr * 4]) = a1;
    *reinterpret_cast<float4 *>(&s_red[1][rg][cgr * 4]) = a2;
    *reinterpret_cast<float4 *>(&s_red[2][rg][cgr * 4]) = ap;
    __syncthreads();
    float4 r1 = make_float4(0.f, 0.f, 0.f, 0.f), r2 = r1;
#pragma unroll
    for (int g = 0; g < RG; ++g) {
        const float4 x = *reinterpret_cast<const float4 *>(&s_red[0][g][cgr * 4]);
        const float4 y = *reinterpret_cast<const float4 *>(&s_red[1][g][cgr * 4]);
        r1.x += x.x; r1.y += x.y; r1.z += x.z; r1.w += x.w;
        r2.x += y.x; r2.y += y.y; r2.z += y.z; r2.w += y.w;
    }
    const float4 wv = *reinterpret_cast<const float4 *>(&s_wv[cgr * 4]);
    const float4 x = make_float4(wv.x - r1.x, wv.y - r1.y, wv.z - r1.z, wv.w - r1.w);
    if (rg == 0) {
        float4 p = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int g = 0; g < RG; ++g) {
            const float4 y = *reinterpret_cast<const float4 *>(&s_red[2][g][cgr * 4]);
            p.x += y.x; p.y += y.y; p.z += y.z; p.w += y.w;
        }
        if (GDN2_IN_BOUNDS(kBufO, o + bh * (long)d_v + j0 + cgr * 4, 4 * sizeof(IO)))
            st_io4<IO>(o + bh * (long)d_v + j0 + cgr * 4, p.x + qk * x.x - qu * r2.x, p.y + qk * x.y - qu * r2.y,
                   p.z + qk * x.z - qu * r2.z, p.w + qk * x.w - qu * r2.w);
    }
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int row = i * RG + rg;
        const float a = s_alpha[row], kr = s_k[row], ur = s_u[row];
        float4 n;
        n.x = a * s[i].x + kr * x.x - ur * r2.x;
        n.y = a * s[i].y + kr * x.y - ur * r2.y;
        n.z = a * s[i].z + kr * x.z - ur * r2.z;
        n.w = a * s[i].w + kr * x.w - ur * r2.w;
        float4 *sp = reinterpret_cast<float4 *>(Sh + (long)row * d_v);
        if (GDN2_IN_BOUNDS(kBufST, sp, 16)) __stcs(sp, n);
    }
}

// Chunk form.  Unrolling the rank-2 edit over a chunk gives the same WY
// algebra as GDN-2 with two pseudo-rows per token, rho = 2 t (key k_t, erase
// b_t.k_t, value w_t.v_t) and rho = 2 t + 1 (direction u_t, erase c_t.u_t,
// value 0), where both rows of a token see the state before that token:
//     A_{rho rho'} = E_rho . K~_rho'  for tok(rho') < tok(rho)     (strict, by token)
//     P_{t rho'}   = Q~_t . K~_rho'   for tok(rho') <= t
//     U = (I + A)^{-1} (V - E S),  O = Q~ S + P U,  S' = diag(Gamma_C)(S + K~^T U)
// with Gamma_t the cumulative decay, Q~ = q.Gamma, K~ = kappa/Gamma, E = eps.Gamma.
// C = 32 tokens make the 64 pseudo-rows of the CUDA-core solve; one block of
// 256 threads per (b, h, 64-column slice of d_v), everything in shared memory.
// A chunk that decays by more than e^-kMaxCudaCoreSpan in some channel runs
// token by token (chunk_token_steps with two pseudo-rows per token) instead.
template <int DK>
struct QedCfg {
    static constexpr int C = 32;        // tokens per chunk
    static constexpr int R = 2 * C;     // pseudo-rows
    static constexpr int NV = 64;
    static constexpr int LK = DK + 1;   // padded strides: [.][DK], [.][R], [.][NV] tiles
    static constexpr int LR = R + 1;
    static constexpr int LV = NV + 1;
    static constexpr int O_Q = 0;                  // [C][LK]  q -> Q~
    static constexpr int O_K = O_Q + C * LK;       // [R][LK]  kappa -> K~
    static constexpr int O_E = O_K + R * LK;       // [R][LK]  erase vectors -> E
    static constexpr int O_G = O_E + R * LK;       // [C][LK]  log-decay, then A [R][LR], P [C][LR]
    static constexpr int G_SIZE = (C * LK > (R + C) * LR) ? C * LK : (R + C) * LR;
    static constexpr int O_T = O_G + G_SIZE;       // [R][LR]
    static constexpr int O_WV = O_T + R * LR;      // [R][LV]  values, then E S
    static constexpr int O_U = O_WV + R * LV;      // [R][LV]
    static constexpr int O_S = O_U + R * LV;       // [DK][LV] state slice
    static constexpr int O_GC = O_S + DK * LV;     // [DK]
    static constexpr int FLOATS = O_GC + DK;
    static constexpr size_t BYTES = sizeof(float) * FLOATS;
};

template <typename IO, int DK>
__global__ void __launch_bounds__(256, 1)
chunk_fwd_qed_kernel(const IO *__restrict__ q, const IO *__restrict__ k, const IO *__restrict__ v,
                     const IO *__restrict__ la, const IO *__restrict__ bg, const IO *__restrict__ cg_,
                     const IO *__restrict__ wg, const float *__restrict__ S0, IO *__restrict__ o,
                     float *__restrict__ S_T, int T, int H, int d_v, float qed_eps) {
    using Cfg = QedCfg<DK>;
    constexpr int C = Cfg::C, R = Cfg::R, NV = Cfg::NV, LK = Cfg::LK, LR = Cfg::LR, LV = Cfg::LV;
    extern __shared__ float sm[];
    float *sQ = sm + Cfg::O_Q, *sK = sm + Cfg::O_K, *sE = sm + Cfg::O_E, *sG = sm + Cfg::O_G;
    float *sA = sG, *sP = sG + R * LR;
    float *sT = sm + Cfg::O_T, *sWV = sm + Cfg::O_WV, *sU = sm + Cfg::O_U, *sS = sm + Cfg::O_S;
    float *sGC = sm + Cfg::O_GC;

    const int tid = threadIdx.x;
    const int j0 = blockIdx.x * NV, h = blockIdx.y, bb = blockIdx.z;
    const long head = (long)bb * H + h;
    const int NC = (T + C - 1) / C;   // the last chunk may be partial (padded rows are zeros)

    for (int idx = tid; idx < DK * NV; idx += 256) {
        const int c = idx / NV, j = idx % NV;
        const float *sp = S0 ? S0 + (head * DK + c) * d_v + j0 + j : nullptr;
        sS[c * LV + j] = (sp && GDN2_IN_BOUNDS(kBufS0, sp, 4)) ? *sp : 0.f;
    }
    for (int n = 0; n < NC; ++n) {
        const long tok0 = (long)bb * T + (long)n * C;
        const int rows = min(C, T - n * C);
        __syncthreads();
        // ---- load; pseudo-row 2t: key k_t, erase b_t.k_t; 2t+1: c_t for now
        for (int idx = tid; idx < C * DK; idx += 256) {
            const int t = idx / DK, c = idx % DK;
            const long g = ((tok0 + t) * H + h) * DK + c;
            const bool in = t < rows;
            const float kv = (in && GDN2_IN_BOUNDS(kBufK, k + g, sizeof(IO))) ? ld_io(k + g) : 0.f;
            sQ[t * LK + c] = (in && GDN2_IN_BOUNDS(kBufQ, q + g, sizeof(IO))) ? ld_io(q + g) : 0.f;
            sK[(2 * t) * LK + c] = kv;
            sE[(2 * t) * LK + c] = (in && GDN2_IN_BOUNDS(kBufB, bg + g, sizeof(IO))) ? ld_io(bg + g) * kv : 0.f;
            sE[(2 * t + 1) * LK + c] = (in && GDN2_IN_BOUNDS(kBufC, cg_ + g, sizeof(IO))) ? ld_io(cg_ + g) : 0.f;
            sG[t * LK + c] = (in && GDN2_IN_BOUNDS(kBufLA, la + g, sizeof(IO))) ? ld_io(la + g) : 0.f;
        }
        for (int idx = tid; idx < C * NV; idx += 256) {
            const int t = idx / NV, j = idx % NV;
            const long g = ((tok0 + t) * H + h) * (long)d_v + j0 + j;
            const bool in = t < rows;
            const float wv = (in && GDN2_IN_BOUNDS(kBufW, wg + g, sizeof(IO))) ? ld_io(wg + g) : 0.f;
            sWV[(2 * t) * LV + j] = (in && GDN2_IN_BOUNDS(kBufV, v + g, sizeof(IO))) ? wv * ld_io(v + g) : 0.f;
            sWV[(2 * t + 1) * LV + j] = 0.f;
        }
        __syncthreads();
        // ---- u_t: warp w takes tokens w, w + 8, ...; lanes stride over the channels
        {
            const int wp = tid >> 5, l = tid & 31;
            for (int t = wp; t < C; t += 8) {
                const float *qr = sQ + t * LK, *kr = sK + (2 * t) * LK;
                float qk = 0.f, kk = 0.f;
                for (int c = l; c < DK; c += 32) {
                    qk = fmaf(qr[c], kr[c], qk);
                    kk = fmaf(kr[c], kr[c], kk);
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    qk += __shfl_xor_sync(0xffffffffu, qk, off);
                    kk += __shfl_xor_sync(0xffffffffu, kk, off);
                }
                const float coef = kk > 0.f ? qk / kk : 0.f;
                float rr = 0.f;
                for (int c = l; c < DK; c += 32) {
                    const float r = qr[c] - coef * kr[c];
                    rr = fmaf(r, r, rr);
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) rr += __shfl_xor_sync(0xffffffffu, rr, off);
                const float den = rr + qed_eps, nu = den > 0.f ? rsqrtf(den) : 0.f;
                float *ur = sK + (2 * t + 1) * LK, *er = sE + (2 * t + 1) * LK;
                for (int c = l; c < DK; c += 32) {
                    const float u = (qr[c] - coef * kr[c]) * nu;
                    ur[c] = u;
                    er[c] *= u;   // c_t . u_t
                }
            }
        }
        __syncthreads();
        // ---- the chunk's decay: past kMaxCudaCoreSpan it runs token by token
        {
            float tot = 0.f;
            if (tid < DK)
                for (int t = 0; t < C; ++t) tot += sG[t * LK + tid];
            if (__syncthreads_or(tid < DK && !(tot >= -kMaxCudaCoreSpan))) {
                // alpha = exp(log_alpha) in place; q . k and q . u per token
                for (int idx = tid; idx < C * DK; idx += 256) {
                    const int t = idx / DK, c = idx % DK;
                    sG[t * LK + c] = __expf(sG[t * LK + c]);
                }
                {
                    const int wp = tid >> 5, l = tid & 31;
                    for (int t = wp; t < C; t += 8) {
                        float qk = 0.f, qu = 0.f;
                        for (int c = l; c < DK; c += 32) {
                            qk = fmaf(sQ[t * LK + c], sK[(2 * t) * LK + c], qk);
                            qu = fmaf(sQ[t * LK + c], sK[(2 * t + 1) * LK + c], qu);
                        }
#pragma unroll
                        for (int off = 16; off > 0; off >>= 1) {
                            qk += __shfl_xor_sync(0xffffffffu, qk, off);
                            qu += __shfl_xor_sync(0xffffffffu, qu, off);
                        }
                        if (l == 0) {
                            sGC[2 * t] = qk;
                            sGC[2 * t + 1] = qu;
                        }
                    }
                }
                __syncthreads();
                chunk_token_steps<DK, NV, 2, IO>(sQ, sK, sE, sG, sWV, sGC, sS, LK, LV, rows, o,
                                                 (tok0 * H + h) * (long)d_v + j0, (long)H * d_v);
                continue;   // the next chunk starts with a barrier
            }
        }
        // ---- cumulative log-decay per channel and the scaled operands
        if (tid < DK) {
            const int c = tid;
            float g = 0.f;
            for (int t = 0; t < C; ++t) {
                g += sG[t * LK + c];
                const float gam = expf(g), inv = expf(-g);
                sQ[t * LK + c] *= gam;
                sE[(2 * t) * LK + c] *= gam;
                sE[(2 * t + 1) * LK + c] *= gam;
                sK[(2 * t) * LK + c] *= inv;
                sK[(2 * t + 1) * LK + c] *= inv;
            }
            sGC[c] = expf(g);
        }
        __syncthreads();
        // ---- A (strict by token) and P (inclusive by token); overwrite the log-decay.
        // Register tiles: A in 4 x 4 (thread: rows 4 (tid / 16).., columns 4 (tid % 16)..),
        // P in 2 x 4; a tile wholly above the token diagonal is zero without work.
        {
            const int rt = tid >> 4, ct = tid & 15;
            float acc[4][4] = {};
            if (ct <= rt) {
                for (int c = 0; c < DK; ++c) {
                    float e[4], kk[4];
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        e[x] = sE[(4 * rt + x) * LK + c];
                        kk[x] = sK[(4 * ct + x) * LK + c];
                    }
#pragma unroll
                    for (int x = 0; x < 4; ++x)
#pragma unroll
                        for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(e[x], kk[y], acc[x][y]);
                }
            }
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) {
                    const int r = 4 * rt + x, i = 4 * ct + y;
                    sA[r * LR + i] = ((i >> 1) < (r >> 1)) ? acc[x][y] : 0.f;
                }
            float pc[2][4] = {};
            if (2 * ct <= 2 * rt + 1) {   // some column token <= some row token
                for (int c = 0; c < DK; ++c) {
                    float qq[2], kk[4];
#pragma unroll
                    for (int x = 0; x < 2; ++x) qq[x] = sQ[(2 * rt + x) * LK + c];
#pragma unroll
                    for (int y = 0; y < 4; ++y) kk[y] = sK[(4 * ct + y) * LK + c];
#pragma unroll
                    for (int x = 0; x < 2; ++x)
#pragma unroll
                        for (int y = 0; y < 4; ++y) pc[x][y] = fmaf(qq[x], kk[y], pc[x][y]);
                }
            }
#pragma unroll
            for (int x = 0; x < 2; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) {
                    const int t = 2 * rt + x, i = 4 * ct + y;
                    sP[t * LR + i] = ((i >> 1) <= t) ? pc[x][y] : 0.f;
                }
        }
        __syncthreads();
        // ---- T = (I + A)^{-1}: column j by 4 threads (rows r = 4 m + qd), right-looking:
        // once row i of the column is final it is broadcast and every later row takes
        // its term; rows above j stay zero by themselves
        {
            const int j = tid >> 2, qd = tid & 3, lane = tid & 31;
            float acc[R / 4];
#pragma unroll
            for (int m = 0; m < R / 4; ++m) acc[m] = (4 * m + qd == j) ? 1.f : 0.f;
#pragma unroll
            for (int i = 0; i < R; ++i) {
                const float xi = __shfl_sync(0xffffffffu, acc[i >> 2], (lane & ~3) | (i & 3));
#pragma unroll
                for (int m = i >> 2; m < R / 4; ++m) {
                    const int r = 4 * m + qd;
                    if (r > i) acc[m] = fmaf(-sA[r * LR + i], xi, acc[m]);
                }
            }
#pragma unroll
            for (int m = 0; m < R / 4; ++m) sT[(4 * m + qd) * LR + j] = acc[m];
        }
        __syncthreads();
        // ---- U = T V - T (E S), 4 x 4 register tiles of the R x NV result
        {
            const int rt = tid >> 4, ct = tid & 15;
            float u1[4][4] = {}, es[4][4] = {};
            for (int i = 0; i < 4 * rt + 4; ++i) {   // T is lower triangular
                float tt[4], vv[4];
#pragma unroll
                for (int x = 0; x < 4; ++x) tt[x] = sT[(4 * rt + x) * LR + i];
#pragma unroll
                for (int y = 0; y < 4; ++y) vv[y] = sWV[i * LV + 4 * ct + y];
#pragma unroll
                for (int x = 0; x < 4; ++x)
#pragma unroll
                    for (int y = 0; y < 4; ++y) u1[x][y] = fmaf(tt[x], vv[y], u1[x][y]);
            }
            for (int c = 0; c < DK; ++c) {
                float e[4], ss[4];
#pragma unroll
                for (int x = 0; x < 4; ++x) e[x] = sE[(4 * rt + x) * LK + c];
#pragma unroll
                for (int y = 0; y < 4; ++y) ss[y] = sS[c * LV + 4 * ct + y];
#pragma unroll
                for (int x = 0; x < 4; ++x)
#pragma unroll
                    for (int y = 0; y < 4; ++y) es[x][y] = fmaf(e[x], ss[y], es[x][y]);
            }
            __syncthreads();   // everyone has read the values before E S replaces them
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) {
                    sU[(4 * rt + x) * LV + 4 * ct + y] = u1[x][y];
                    sWV[(4 * rt + x) * LV + 4 * ct + y] = es[x][y];
                }
            __syncthreads();
            for (int i = 0; i < 4 * rt + 4; ++i) {
                float tt[4], vv[4];
#pragma unroll
                for (int x = 0; x < 4; ++x) tt[x] = sT[(4 * rt + x) * LR + i];
#pragma unroll
                for (int y = 0; y < 4; ++y) vv[y] = sWV[i * LV + 4 * ct + y];
#pragma unroll
                for (int x = 0; x < 4; ++x)
#pragma unroll
                    for (int y = 0; y < 4; ++y) u1[x][y] = fmaf(-tt[x], vv[y], u1[x][y]);
            }
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) sU[(4 * rt + x) * LV + 4 * ct + y] = u1[x][y];
        }
        __syncthreads();
        // ---- O = Q~ S + P U on the token rows, 2 x 4 register tiles
        {
            const int rt = tid >> 4, ct = tid & 15;
            float ov[2][4] = {};
            for (int c = 0; c < DK; ++c) {
                float qq[2], ss[4];
#pragma unroll
                for (int x = 0; x < 2; ++x) qq[x] = sQ[(2 * rt + x) * LK + c];
#pragma unroll
                for (int y = 0; y < 4; ++y) ss[y] = sS[c * LV + 4 * ct + y];
#pragma unroll
                for (int x = 0; x < 2; ++x)
#pragma unroll
                    for (int y = 0; y < 4; ++y) ov[x][y] = fmaf(qq[x], ss[y], ov[x][y]);
            }
            for (int i = 0; i < 4 * rt + 4; ++i) {   // P is zero past the row's token
                float pp[2], uu[4];
#pragma unroll
                for (int x = 0; x < 2; ++x) pp[x] = sP[(2 * rt + x) * LR + i];
#pragma unroll
                for (int y = 0; y < 4; ++y) uu[y] = sU[i * LV + 4 * ct + y];
#pragma unroll
                for (int x = 0; x < 2; ++x)
#pragma unroll
                    for (int y = 0; y < 4; ++y) ov[x][y] = fmaf(pp[x], uu[y], ov[x][y]);
            }
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                const int t = 2 * rt + x;
                if (t < rows) {
                    const long g = ((tok0 + t) * H + h) * (long)d_v + j0 + 4 * ct;
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
        // ---- S <- diag(Gamma_C) (S + K~^T U), 4 x 8 register tiles of the DK x NV state
        for (int tile = tid; tile < (DK / 4) * (NV / 8); tile += 256) {
            const int rt = tile / (NV / 8), ct = tile % (NV / 8);
            float sv[4][8];
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 8; ++y) sv[x][y] = sS[(4 * rt + x) * LV + 8 * ct + y];
            for (int i = 0; i < R; ++i) {
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
