// chunk_tc.cuh -- chunk-parallel GDN-2 forward on sm_100a tensor cores.
//
// Chunk algebra (the burn-gdn2 README recurrence, "Architecture" section,
// regrouped over chunks of C = 64 tokens as in its "Chunk WY (train)" mode):
//     A = strict_lower(E K~^T),  P = lower(Q~ K~^T),  T = (I + A)^{-1},
//     U = T (W.V) - (T E) S,     O = Q~ S + P U,      S' = diag(gamma_C)(S + K~^T U)
// with Q~ = Q.Gamma, K~ = K/Gamma, E = B.K.Gamma, Gamma_r = exp(cumsum_{s<=r} log_alpha_s)
// per key channel, and S the fp32 state at the chunk start.
//
// One CTA (256 threads) owns one (b, h, NV-column slice of d_v) and walks
// the T/64 chunks in order as a two-stage software pipeline:
//   key warpgroup   (threads   0-127), chunk m: everything that does not
//                   depend on the state --
//       prep   16-byte loads of log_alpha, q, k, b from L2 (TMA L2 prefetch
//              a few chunks ahead); per-channel cumulative log-decay with a
//              cross-thread scan; bf16 MMA operands Q~^T, E^T, K~^T written
//              as rows c of 128B-swizzled tiles; W.V for this column slice.
//       MMA1   [Q~; E] K~^T -> TMEM (rows 0-63 P', rows 64-127 A')
//       solve  T = (I + A)^{-1} in fp32 (16x16 diagonal blocks by forward
//              substitution, off-diagonal blocks by vectorised block products)
//       MMA2   (T E)^T = E^T T^T -> TMEM -> bf16 (T E)^T tile
//       MMA3   [. ; T] (W.V)     -> TMEM rows 64-127 = T (W.V)
//   chain warpgroup (threads 128-255), chunk m-1: the sequential state pass --
//       MMA_s  [Q~; T E] S -> X (rows 0-63 Q~ S, rows 64-127 T E S)
//       U      = T (W.V) - T E S   (bf16 into shared memory)
//       MMA_u  S += K~^T U   (fp32 state stays in TMEM across chunks)
//       MMA_o  X += [P; .] U (rows 0-63: O = Q~ S + P U)
//       out    S rows *= gamma_C (bf16 copy for the next MMA_s), O rows -> HBM
// Operands that cross the two warpgroups (Q~, K~, P, gamma_C) are double
// buffered; (T E)^T and T (W.V) are single buffered and handed over with an
// mbarrier.  All MMAs are tcgen05.mma kind::f16, M = 128 (bf16 x bf16 ->
// fp32); each warpgroup issues its own from one thread and tracks them with
// tcgen05.commit.  Every mbarrier wait is bounded; a timeout aborts cleanly.
#pragma once
#include "gdn2_device.cuh"

namespace gdn2 {

template <int DK, int NV>
struct TcCfg {
    static_assert(DK == 64 || DK == 128, "d_k");
    static_assert(NV == 64 || NV == 128, "value slice");
    static constexpr int C = 64;
    // 128-row x 64-column bf16 tiles (16 KB), 128B swizzle
    static constexpr uint32_t OFF_Q0 = 0;             // Q~^T  [c][r], stage 0
    static constexpr uint32_t OFF_Q1 = 16384;         // Q~^T  [c][r], stage 1
    static constexpr uint32_t OFF_ET = 32768;         // (T E)^T [c][r]
    static constexpr uint32_t OFF_E = 49152;          // E^T   [c][r]
    static constexpr uint32_t OFF_K0 = 65536;         // K~^T  [c][i], stage 0
    static constexpr uint32_t OFF_K1 = 81920;         // K~^T  [c][i], stage 1
    // 64-row x 64-column bf16 tiles (8 KB)
    static constexpr uint32_t OFF_P0 = 98304;         // P [r][i], stage 0
    static constexpr uint32_t OFF_T = 106496;         // T [r][i]   (P0 + 8 KB)
    static constexpr uint32_t OFF_P1 = 114688;        // P [r][i], stage 1
    static constexpr uint32_t OFF_WV = 122880;        // W.V [jb][i][64]   (P1 + 8 KB)
    static constexpr uint32_t OFF_S = OFF_WV + (NV / 64) * 8192u;    // bf16 S [jb][c][64]
    static constexpr uint32_t OFF_U = OFF_S + (NV / 64) * 16384u;    // U [jb][i][64]
    static constexpr uint32_t OFF_SCR = OFF_U + (NV / 64) * 8192u;   // fp32 A/T [64][68] + W [16][48]
    static constexpr int LDA = 68;
    static constexpr uint32_t OFF_TOT = OFF_SCR + (64 * LDA + 16 * 48) * 4;   // scan totals
    static constexpr uint32_t OFF_GC = OFF_TOT + 4096;                          // gamma_C [2][128]
    static constexpr uint32_t OFF_BAR = OFF_GC + 1024;
    static constexpr uint32_t OFF_TMEMP = OFF_BAR + 128;
    static constexpr uint32_t SMEM_BYTES = OFF_TMEMP + 16;
    static constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;
    // TMEM columns: [AP / (TE)^T 64][T W.V  NV][X NV][S NV]
    static constexpr uint32_t T_AP = 0, T_UT = 64, T_X = 64 + NV, T_S = 64 + 2 * NV;
    static constexpr uint32_t TMEM_COLS = (64 + 3 * NV) <= 256 ? 256 : 512;
    static constexpr int PREFETCH = 3;
    // prep thread tiling: 8 channels x RPT rows per thread
    static constexpr int CG = DK / 8, RG = 128 / CG, RPT = 64 / RG;
};

__device__ __forceinline__ void named_bar(int id) {
    asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory");
}
// Barrier over one warpgroup that also ORs a predicate across it.
__device__ __forceinline__ bool wg_any(int id, bool p) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.or.pred po, %2, 128, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(p)), "r"(id)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ uint4 ldg_u4(const __nv_bfloat16 *p) {
    return __ldg(reinterpret_cast<const uint4 *>(p));
}
// bf16 element `ch` (0..7) of a 16-byte vector; `ch` folds to a constant
// once the caller's loop is unrolled.
__device__ __forceinline__ float bf16_get(const uint4 &u, int ch) {
    const uint32_t w = (ch >> 1) == 0 ? u.x : (ch >> 1) == 1 ? u.y : (ch >> 1) == 2 ? u.z : u.w;
    return (ch & 1) ? bf16_hi(w) : bf16_lo(w);
}

// Off-diagonal block row IB of T = (I + A)^{-1} (A strictly lower, 64x64,
// fp32 in sA with row stride LDA; rows above 16*IB already hold T, the
// diagonal blocks hold their inverses D):
//     W         = A[16IB:16IB+16, :16IB] T[:16IB, :16IB]
//     T[16IB:16IB+16, :16IB] = -D_IB W
template <int IB, int LDA>
__device__ __forceinline__ void solve_block_row(float *sA, float *sW, int t) {
    constexpr int N = 16 * IB, NC4 = N / 4;
    const int r = t >> 3, c4 = t & 7;
#pragma unroll
    for (int mm = 0; mm < (NC4 + 7) / 8; ++mm) {
        const int col4 = c4 + 8 * mm;
        if (col4 < NC4) {
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            const float *arow = sA + (N + r) * LDA;
#pragma unroll
            for (int kk = 0; kk < N; ++kk) {
                const float a = arow[kk];
                const float4 tv = *reinterpret_cast<const float4 *>(sA + kk * LDA + 4 * col4);
                acc.x = fmaf(a, tv.x, acc.x); acc.y = fmaf(a, tv.y, acc.y);
                acc.z = fmaf(a, tv.z, acc.z); acc.w = fmaf(a, tv.w, acc.w);
            }
            *reinterpret_cast<float4 *>(sW + r * 48 + 4 * col4) = acc;
        }
    }
    named_bar(1);
#pragma unroll
    for (int mm = 0; mm < (NC4 + 7) / 8; ++mm) {
        const int col4 = c4 + 8 * mm;
        if (col4 < NC4) {
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            const float *drow = sA + (N + r) * LDA + N;
#pragma unroll
            for (int ss = 0; ss < 16; ++ss) {
                const float dv = drow[ss];
                const float4 wv = *reinterpret_cast<const float4 *>(sW + ss * 48 + 4 * col4);
                acc.x = fmaf(dv, wv.x, acc.x); acc.y = fmaf(dv, wv.y, acc.y);
                acc.z = fmaf(dv, wv.z, acc.z); acc.w = fmaf(dv, wv.w, acc.w);
            }
            *reinterpret_cast<float4 *>(sA + (N + r) * LDA + 4 * col4) = make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
        }
    }
    named_bar(1);
}

template <int DK, int NV>
__global__ void __launch_bounds__(256, 1)
chunk_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_la, const __grid_constant__ CUtensorMap tm_b,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_w,
                    const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                    const __nv_bfloat16 *__restrict__ v, const __nv_bfloat16 *__restrict__ la,
                    const __nv_bfloat16 *__restrict__ bg, const __nv_bfloat16 *__restrict__ wg,
                    const float *__restrict__ S0, __nv_bfloat16 *__restrict__ o, float *__restrict__ S_T,
                    int T, int H, int d_v, unsigned long long wait_ns) {
    using Cfg = TcCfg<DK, NV>;
    constexpr int LDA = Cfg::LDA;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(smem);

    const int tid = threadIdx.x, warp = tid >> 5;
    const int j0 = blockIdx.x * NV, h = blockIdx.y, bb = blockIdx.z;
    const int NC = T / Cfg::C;
    const long head = (long)bb * H + h;
    const long row0 = (long)bb * T;   // token index of t = 0 for this batch row

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
    uint64_t *bk1 = bars + 0, *bk2 = bars + 1;                 // key: MMA1, MMA2+3 done
    uint64_t *bc1 = bars + 2, *bc2 = bars + 3, *bc3 = bars + 4; // chain: MMA_s, MMA_u, MMA_o done
    uint64_t *full = bars + 5;                                 // [2] key products of a chunk ready
    uint64_t *empty = bars + 7;                                // [2] chain done with a stage
    uint64_t *utfree = bars + 9;                               // chain read T(W.V), MMA_s done
    uint64_t *drain = bars + 10;                               // [2] teardown
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + Cfg::OFF_TMEMP);
    float *gC = reinterpret_cast<float *>(smem + Cfg::OFF_GC);
    float *sA = reinterpret_cast<float *>(smem + Cfg::OFF_SCR);
    float *sW = sA + 64 * LDA;
    float *sTot = reinterpret_cast<float *>(smem + Cfg::OFF_TOT);

    // ---------------------------------------------------------------- setup
    for (uint32_t off = tid * 16u; off < Cfg::OFF_SCR; off += 256u * 16u) st_shared_v4(sb + off, 0u, 0u, 0u, 0u);
    if (tid == 0) {
        for (int i = 0; i < 12; ++i) mbar_init(bars + i, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_holder, Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const uint32_t lane_q = static_cast<uint32_t>((warp & 3) * 32) << 16;   // this warp's TMEM lanes
    const uint32_t t_AP = tmem + Cfg::T_AP, t_UT = tmem + Cfg::T_UT;
    const uint32_t t_X = tmem + Cfg::T_X, t_S = tmem + Cfg::T_S;
    bool failed = false;

    if (tid < 128) {
        // ============================================================ key side
        const int t = tid;
        auto prefetch = [&](int n) {
            const int r = static_cast<int>(row0) + n * 64;
            for (int kb = 0; kb < DK / 64; ++kb) {
                tma_prefetch_l2_3d(&tm_la, kb * 64, h, r);
                tma_prefetch_l2_3d(&tm_q, kb * 64, h, r);
                tma_prefetch_l2_3d(&tm_k, kb * 64, h, r);
                tma_prefetch_l2_3d(&tm_b, kb * 64, h, r);
            }
            for (int vb = 0; vb < NV / 64; ++vb) {
                tma_prefetch_l2_3d(&tm_v, j0 + vb * 64, h, r);
                tma_prefetch_l2_3d(&tm_w, j0 + vb * 64, h, r);
            }
        };
        if (t == 0)
            for (int p = 0; p < Cfg::PREFETCH && p < NC; ++p) prefetch(p);
        const int rg = t % Cfg::RG, cg = t / Cfg::RG;   // prep tile: rows rg*RPT.., channels 8cg..
        uint32_t ph1 = 0, ph2 = 0;
        for (int m = 0; m < NC; ++m) {
            const int s = m & 1;
            const uint32_t u = static_cast<uint32_t>(m >> 1);
            if (t == 0 && m + Cfg::PREFETCH < NC) prefetch(m + Cfg::PREFETCH);
            if (m >= 2) {
                const bool ok = mbar_wait(&empty[s], (u - 1u) & 1u, wait_ns);
                if (wg_any(1, !ok)) { failed = true; break; }
            }
            const uint32_t OQ = s ? Cfg::OFF_Q1 : Cfg::OFF_Q0, OK = s ? Cfg::OFF_K1 : Cfg::OFF_K0;
            const uint32_t OP = s ? Cfg::OFF_P1 : Cfg::OFF_P0;
            // ---------------------------------------------------------- prep
            {
                constexpr int RPT = Cfg::RPT;
                const long tok = row0 + (long)m * 64 + rg * RPT;
                uint4 xla[RPT], xq[RPT], xk[RPT], xb[RPT];
#pragma unroll
                for (int e = 0; e < RPT; ++e) {
                    const long off = ((tok + e) * H + h) * DK + 8 * cg;
                    xla[e] = ldg_u4(la + off);
                    xq[e] = ldg_u4(q + off);
                    xk[e] = ldg_u4(k + off);
                    xb[e] = ldg_u4(bg + off);
                }
                // per-channel sums of this thread's rows, then an exclusive scan over row groups
                {
                    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int e = 0; e < RPT; ++e)
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch) acc[ch] += bf16_get(xla[e], ch);
                    float4 *tp = reinterpret_cast<float4 *>(sTot + rg * DK + 8 * cg);
                    tp[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
                    tp[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
                }
                named_bar(1);
                float off8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                for (int r2 = 0; r2 < rg; ++r2) {
                    const float4 a = *reinterpret_cast<const float4 *>(sTot + r2 * DK + 8 * cg);
                    const float4 b4 = *reinterpret_cast<const float4 *>(sTot + r2 * DK + 8 * cg + 4);
                    off8[0] += a.x; off8[1] += a.y; off8[2] += a.z; off8[3] += a.w;
                    off8[4] += b4.x; off8[5] += b4.y; off8[6] += b4.z; off8[7] += b4.w;
                }
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const int c = 8 * cg + ch;
                    uint32_t pq[RPT / 2], pe[RPT / 2], pk[RPT / 2];
                    float gg = off8[ch];
#pragma unroll
                    for (int e = 0; e < RPT; e += 2) {
                        const float g0 = gg + bf16_get(xla[e], ch);
                        const float g1 = g0 + bf16_get(xla[e + 1], ch);
                        gg = g1;
                        const float ga0 = __expf(g0), ga1 = __expf(g1);
                        const float iv0 = __expf(-g0), iv1 = __expf(-g1);
                        const float k0 = bf16_get(xk[e], ch), k1 = bf16_get(xk[e + 1], ch);
                        pq[e / 2] = pack_bf16x2(bf16_get(xq[e], ch) * ga0, bf16_get(xq[e + 1], ch) * ga1);
                        pe[e / 2] = pack_bf16x2(bf16_get(xb[e], ch) * k0 * ga0, bf16_get(xb[e + 1], ch) * k1 * ga1);
                        pk[e / 2] = pack_bf16x2(k0 * iv0, k1 * iv1);
                    }
                    if constexpr (RPT == 8) {
                        const uint32_t co = sw128_chunk(c, rg);
                        st_shared_v4(sb + OQ + co, pq[0], pq[1], pq[2], pq[3]);
                        st_shared_v4(sb + Cfg::OFF_E + co, pe[0], pe[1], pe[2], pe[3]);
                        st_shared_v4(sb + OK + co, pk[0], pk[1], pk[2], pk[3]);
                    } else {
                        const uint32_t co = sw128_chunk(c, rg >> 1) + (rg & 1) * 8;
                        asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(sb + OQ + co), "r"(pq[0]), "r"(pq[1]) : "memory");
                        asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(sb + Cfg::OFF_E + co), "r"(pe[0]), "r"(pe[1]) : "memory");
                        asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(sb + OK + co), "r"(pk[0]), "r"(pk[1]) : "memory");
                    }
                    if (rg == Cfg::RG - 1) gC[s * 128 + c] = __expf(gg);
                }
                if (DK < 128 && t < 128 - DK) gC[s * 128 + DK + t] = 1.f;
            }
            fence_proxy_async_smem();
            named_bar(1);
            // ---------------------------------------------------------- MMA1
            if (t == 0) {
                tc_fence_after();
                const uint32_t id1 = idesc_bf16(128, 64, true, true);
#pragma unroll
                for (int ks = 0; ks < DK / 16; ++ks)
                    umma_bf16(t_AP, sdesc_sw128(sb + OQ + ks * 2048, Cfg::OFF_E - OQ, 1024),
                              sdesc_sw128(sb + OK + ks * 2048, 8192, 1024), id1, ks > 0 ? 1u : 0u);
                umma_commit(bk1);
            }
            // W.V for this column slice while MMA1 runs
            {
                constexpr int CPR = NV / 8;                 // 16-byte chunks per row
                constexpr int IT = 64 * CPR / 128;          // chunks per thread
                uint4 xv[IT], xw[IT];
#pragma unroll
                for (int it = 0; it < IT; ++it) {
                    const int i = t + it * 128, r = i / CPR, jc = i % CPR;
                    const long off = ((row0 + (long)m * 64 + r) * H + h) * d_v + j0 + jc * 8;
                    xv[it] = ldg_u4(v + off);
                    xw[it] = ldg_u4(wg + off);
                }
#pragma unroll
                for (int it = 0; it < IT; ++it) {
                    const int i = t + it * 128, r = i / CPR, jc = i % CPR;
                    const uint4 a = xv[it], b4 = xw[it];
                    st_shared_v4(sb + Cfg::OFF_WV + (jc >> 3) * 8192u + sw128_chunk(r, jc & 7),
                                 pack_bf16x2(bf16_lo(a.x) * bf16_lo(b4.x), bf16_hi(a.x) * bf16_hi(b4.x)),
                                 pack_bf16x2(bf16_lo(a.y) * bf16_lo(b4.y), bf16_hi(a.y) * bf16_hi(b4.y)),
                                 pack_bf16x2(bf16_lo(a.z) * bf16_lo(b4.z), bf16_hi(a.z) * bf16_hi(b4.z)),
                                 pack_bf16x2(bf16_lo(a.w) * bf16_lo(b4.w), bf16_hi(a.w) * bf16_hi(b4.w)));
                }
            }
            fence_proxy_async_smem();
            {
                const bool ok = mbar_wait(bk1, ph1, wait_ns);
                ph1 ^= 1u;
                if (wg_any(1, !ok)) { failed = true; break; }
            }
            tc_fence_after();
            // ------------------------------------------- read out P' and A
            if (warp < 2) {
                const int r = t;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float x[32];
                    tmem_ld32(t_AP + lane_q + half * 32, x);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        uint32_t p[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int i = half * 32 + q4 * 8 + 2 * e;
                            p[e] = pack_bf16x2(i <= r ? x[q4 * 8 + 2 * e] : 0.f, i + 1 <= r ? x[q4 * 8 + 2 * e + 1] : 0.f);
                        }
                        st_shared_v4(sb + OP + sw128_chunk(r, half * 4 + q4), p[0], p[1], p[2], p[3]);
                    }
                }
            } else {
                const int r = t - 64;
                float *arow = sA + r * LDA;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float x[32];
                    tmem_ld32(t_AP + lane_q + half * 32, x);
#pragma unroll
                    for (int e = 0; e < 32; e += 4) {
                        const int i = half * 32 + e;
                        *reinterpret_cast<float4 *>(arow + i) =
                            make_float4(i < r ? x[e] : 0.f, i + 1 < r ? x[e + 1] : 0.f, i + 2 < r ? x[e + 2] : 0.f,
                                        i + 3 < r ? x[e + 3] : 0.f);
                    }
                }
            }
            tc_fence_before();
            named_bar(1);
            // ------------------------------------------ T = (I + A)^{-1}
            {
                float xd[16];
                const int dR = (t >> 4) * 16, dj = t & 15;
                if (t < 64) {
#pragma unroll
                    for (int r = 0; r < 16; ++r) {
                        float acc = (r == dj) ? 1.f : 0.f;
#pragma unroll
                        for (int i = 0; i < r; ++i) acc = fmaf(-sA[(dR + r) * LDA + dR + i], xd[i], acc);
                        xd[r] = acc;
                    }
                }
                named_bar(1);
                if (t < 64) {
#pragma unroll
                    for (int r = 0; r < 16; ++r) sA[(dR + r) * LDA + dR + dj] = xd[r];
                }
                named_bar(1);
            }
            solve_block_row<1, LDA>(sA, sW, t);
            solve_block_row<2, LDA>(sA, sW, t);
            solve_block_row<3, LDA>(sA, sW, t);
#pragma unroll
            for (int idx = t; idx < 512; idx += 128) {
                const int r = idx >> 3, ch = idx & 7;
                const float4 a = *reinterpret_cast<const float4 *>(sA + r * LDA + ch * 8);
                const float4 b4 = *reinterpret_cast<const float4 *>(sA + r * LDA + ch * 8 + 4);
                st_shared_v4(sb + Cfg::OFF_T + sw128_chunk(r, ch), pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w),
                             pack_bf16x2(b4.x, b4.y), pack_bf16x2(b4.z, b4.w));
            }
            fence_proxy_async_smem();
            // the chain must have read T(W.V) and run MMA_s of the previous chunk
            if (m >= 1) {
                const bool ok = mbar_wait(utfree, static_cast<uint32_t>((m - 1) & 1), wait_ns);
                if (wg_any(1, !ok)) { failed = true; break; }
            } else {
                named_bar(1);
            }
            // ------------------------------------------------ MMA2 + MMA3
            if (t == 0) {
                tc_fence_after();
                const uint32_t id2 = idesc_bf16(128, 64, false, false);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_bf16(t_AP, sdesc_sw128(sb + Cfg::OFF_E + ks * 32, 16, 1024),
                              sdesc_sw128(sb + Cfg::OFF_T + ks * 32, 16, 1024), id2, ks > 0 ? 1u : 0u);
                const uint32_t id3 = idesc_bf16(128, NV, false, true);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_bf16(t_UT, sdesc_sw128(sb + Cfg::OFF_P0 + ks * 32, 16, 1024),
                              sdesc_sw128(sb + Cfg::OFF_WV + ks * 2048, 8192, 1024), id3, ks > 0 ? 1u : 0u);
                umma_commit(bk2);
            }
            {
                const bool ok = mbar_wait(bk2, ph2, wait_ns);
                ph2 ^= 1u;
                if (wg_any(1, !ok)) { failed = true; break; }
            }
            tc_fence_after();
            // (T E)^T rows c -> bf16 tile
            {
                const int c = t;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float x[32];
                    tmem_ld32(t_AP + lane_q + half * 32, x);
                    if (c < DK) {
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4)
                            st_shared_v4(sb + Cfg::OFF_ET + sw128_chunk(c, half * 4 + q4),
                                         pack_bf16x2(x[8 * q4], x[8 * q4 + 1]), pack_bf16x2(x[8 * q4 + 2], x[8 * q4 + 3]),
                                         pack_bf16x2(x[8 * q4 + 4], x[8 * q4 + 5]),
                                         pack_bf16x2(x[8 * q4 + 6], x[8 * q4 + 7]));
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar(1);
            if (t == 0) mbar_arrive(&full[s]);
        }
        if (t == 0) {   // wait (bounded) for this issuer's MMAs before teardown
            umma_commit(&drain[0]);
            mbar_wait(&drain[0], 0u, wait_ns);
        }
    } else {
        // ========================================================== chain side
        const int t = tid - 128;
        // initial state: fp32 into TMEM (lane c = key channel), bf16 copy
        {
            const int c = t;
            for (int jc = 0; jc < NV / 32; ++jc) {
                float sv[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) sv[e] = 0.f;
                if (S0 != nullptr && c < DK) {
                    const float4 *src = reinterpret_cast<const float4 *>(S0 + (head * DK + c) * d_v + j0 + jc * 32);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float4 x = src[e];
                        sv[4 * e] = x.x; sv[4 * e + 1] = x.y; sv[4 * e + 2] = x.z; sv[4 * e + 3] = x.w;
                    }
                }
                tmem_st32(t_S + lane_q + jc * 32, sv);
                const uint32_t tile = sb + Cfg::OFF_S + ((jc * 32) >> 6) * 16384u;
                const uint32_t ch0 = ((jc * 32) & 63) >> 3;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4)
                    st_shared_v4(tile + sw128_chunk(c, ch0 + q4), pack_bf16x2(sv[8 * q4], sv[8 * q4 + 1]),
                                 pack_bf16x2(sv[8 * q4 + 2], sv[8 * q4 + 3]), pack_bf16x2(sv[8 * q4 + 4], sv[8 * q4 + 5]),
                                 pack_bf16x2(sv[8 * q4 + 6], sv[8 * q4 + 7]));
            }
            tmem_st_wait();
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar(2);
        }
        uint32_t ph1 = 0, ph2 = 0, ph3 = 0;
        for (int n = 0; n < NC; ++n) {
            const int s = n & 1;
            const uint32_t u = static_cast<uint32_t>(n >> 1);
            const uint32_t OQ = s ? Cfg::OFF_Q1 : Cfg::OFF_Q0, OK = s ? Cfg::OFF_K1 : Cfg::OFF_K0;
            const uint32_t OP = s ? Cfg::OFF_P1 : Cfg::OFF_P0;
            {
                const bool ok = mbar_wait(&full[s], u & 1u, wait_ns);
                if (wg_any(2, !ok)) { failed = true; break; }
            }
            // ------------------------------------------------------ MMA_s
            if (t == 0) {
                tc_fence_after();
                const uint32_t ids = idesc_bf16(128, NV, true, true);
#pragma unroll
                for (int ks = 0; ks < DK / 16; ++ks)
                    umma_bf16(t_X, sdesc_sw128(sb + OQ + ks * 2048, Cfg::OFF_ET - OQ, 1024),
                              sdesc_sw128(sb + Cfg::OFF_S + ks * 2048, 16384, 1024), ids, ks > 0 ? 1u : 0u);
                umma_commit(bc1);
            }
            {
                const bool ok = mbar_wait(bc1, ph1, wait_ns);
                ph1 ^= 1u;
                if (wg_any(2, !ok)) { failed = true; break; }
            }
            tc_fence_after();
            if (warp >= 6) {
                const int r = t - 64;   // U row r (TMEM lanes 64-127)
#pragma unroll 1
                for (int jc = 0; jc < NV / 32; ++jc) {
                    float x[32], ut[32];
                    tmem_ld32(t_X + lane_q + jc * 32, x);
                    tmem_ld32(t_UT + lane_q + jc * 32, ut);
                    const uint32_t tile = sb + Cfg::OFF_U + ((jc * 32) >> 6) * 8192u;
                    const uint32_t ch0 = ((jc * 32) & 63) >> 3;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const int e = 8 * q4;
                        st_shared_v4(tile + sw128_chunk(r, ch0 + q4), pack_bf16x2(ut[e] - x[e], ut[e + 1] - x[e + 1]),
                                     pack_bf16x2(ut[e + 2] - x[e + 2], ut[e + 3] - x[e + 3]),
                                     pack_bf16x2(ut[e + 4] - x[e + 4], ut[e + 5] - x[e + 5]),
                                     pack_bf16x2(ut[e + 6] - x[e + 6], ut[e + 7] - x[e + 7]));
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar(2);
            // ---------------------------------------------- MMA_u and MMA_o
            if (t == 0) {
                mbar_arrive(utfree);
                tc_fence_after();
                const uint32_t idu = idesc_bf16(128, NV, false, true);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_bf16(t_S, sdesc_sw128(sb + OK + ks * 32, 16, 1024),
                              sdesc_sw128(sb + Cfg::OFF_U + ks * 2048, 8192, 1024), idu, 1u);
                umma_commit(bc2);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_bf16(t_X, sdesc_sw128(sb + OP + ks * 32, 16, 1024),
                              sdesc_sw128(sb + Cfg::OFF_U + ks * 2048, 8192, 1024), idu, 1u);
                umma_commit(bc3);
            }
            {
                const bool ok = mbar_wait(bc2, ph2, wait_ns);
                ph2 ^= 1u;
                if (wg_any(2, !ok)) { failed = true; break; }
            }
            tc_fence_after();
            {
                const int c = t;
                const float gcv = gC[s * 128 + c];
                const bool last = (n + 1 == NC);
#pragma unroll 1
                for (int jc = 0; jc < NV / 32; ++jc) {
                    float sv[32];
                    tmem_ld32(t_S + lane_q + jc * 32, sv);
#pragma unroll
                    for (int e = 0; e < 32; ++e) sv[e] *= gcv;
                    tmem_st32(t_S + lane_q + jc * 32, sv);
                    if (c < DK) {
                        const uint32_t tile = sb + Cfg::OFF_S + ((jc * 32) >> 6) * 16384u;
                        const uint32_t ch0 = ((jc * 32) & 63) >> 3;
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const int e = 8 * q4;
                            st_shared_v4(tile + sw128_chunk(c, ch0 + q4), pack_bf16x2(sv[e], sv[e + 1]),
                                         pack_bf16x2(sv[e + 2], sv[e + 3]), pack_bf16x2(sv[e + 4], sv[e + 5]),
                                         pack_bf16x2(sv[e + 6], sv[e + 7]));
                        }
                        if (last && S_T != nullptr) {
                            float4 *dst = reinterpret_cast<float4 *>(S_T + (head * DK + c) * d_v + j0 + jc * 32);
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                dst[e] = make_float4(sv[4 * e], sv[4 * e + 1], sv[4 * e + 2], sv[4 * e + 3]);
                        }
                    }
                }
            }
            {
                const bool ok = mbar_wait(bc3, ph3, wait_ns);
                ph3 ^= 1u;
                if (wg_any(2, !ok)) { failed = true; break; }
            }
            tc_fence_after();
            if (warp == 4 || warp == 5) {
                const int r = t;   // output row r (TMEM lanes 0-63)
                __nv_bfloat16 *orow = o + ((row0 + (long)n * 64 + r) * H + h) * (long)d_v + j0;
#pragma unroll 1
                for (int jc = 0; jc < NV / 32; ++jc) {
                    float x[32];
                    tmem_ld32(t_X + lane_q + jc * 32, x);
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + jc * 32);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const int e = 8 * q4;
                        dst[q4] = make_uint4(pack_bf16x2(x[e], x[e + 1]), pack_bf16x2(x[e + 2], x[e + 3]),
                                             pack_bf16x2(x[e + 4], x[e + 5]), pack_bf16x2(x[e + 6], x[e + 7]));
                    }
                }
            }
            tmem_st_wait();
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar(2);
            if (t == 0) mbar_arrive(&empty[s]);
        }
        if (t == 0) {
            umma_commit(&drain[1]);
            mbar_wait(&drain[1], 0u, wait_ns);
        }
    }

    // ------------------------------------------------------------- teardown
    const bool any_failed = __syncthreads_or(failed);
    if (any_failed && tid == 0) record_timeout();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, Cfg::TMEM_COLS);
    }
}

}  // namespace gdn2
