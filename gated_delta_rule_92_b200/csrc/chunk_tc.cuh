// chunk_tc.cuh -- chunk-parallel GDN-2 forward on sm_100a tensor cores.
//
// Same chunk algebra as the CUDA-core kernel (chunk_ffma.cuh), from the
// burn-gdn2 README recurrence ("Architecture"; "Chunk WY (train)" mode):
//     A = strict_lower(E K~^T),  P = lower(Q~ K~^T),  T = (I + A)^{-1},
//     U = T (W.V) - (T E) S,     O = Q~ S + P U,      S' = diag(gamma_C)(S + K~^T U)
// with Q~ = Q.Gamma, K~ = K/Gamma, E = B.K.Gamma and Gamma_r = exp(cumsum log_alpha).
//
// One CTA (4 warps) owns one (b, h, NV-column slice of d_v) and walks the
// T/64 chunks in order.  Per chunk:
//   TMA      q, k, log_alpha, b, v, w tiles -> shared memory (128B swizzle);
//            tiles a few chunks ahead are prefetched into L2.
//   prep     thread c scans key channel c: g, gamma, and writes the bf16 MMA
//            operands Q~^T, E^T, K~^T as rows c of 128B-swizzled tiles;
//            W.V is formed in place in the v tile.
//   MMA1     [Q~; E] K~^T  -> TMEM (M=128: rows 0-63 P', rows 64-127 A').
//   solve    T = (I + A)^{-1} in fp32 on CUDA cores (16x16 blocked
//            forward substitution), written as bf16 next to P: TP = [P; T].
//   MMA2     (T E)^T = E^T T^T -> TMEM, copied back over E as bf16.
//   MMA3     [P; T] (W.V)      -> TMEM (rows 64-127 = T W.V).
//   MMA_s    [Q~; T E] S       -> TMEM X (rows 0-63 Q~S, rows 64-127 T E S).
//   U        = T W.V - T E S   (rows 64-127), bf16 into shared memory.
//   MMA_u    S += K~^T U  (fp32 state stays in TMEM across chunks)
//   MMA_o    X += [P; T] U    (rows 0-63: O = Q~S + P U; rows 64-127 unused)
//   out      O rows -> global (bf16); S rows *= gamma_C, bf16 copy -> shared
//            memory for the next chunk's MMA_s; S_T after the last chunk.
// All MMAs are tcgen05.mma kind::f16 (bf16 x bf16 -> fp32), M = 128, issued
// by one thread; completion is tracked with tcgen05.commit -> mbarrier.
// Every mbarrier wait is bounded; a timeout aborts the CTA cleanly.
#pragma once
#include "gdn2_device.cuh"

namespace gdn2 {

template <int DK, int NV>
struct TcCfg {
    static_assert(DK == 64 || DK == 128, "d_k");
    static_assert(NV == 64 || NV == 128, "value slice");
    static constexpr int C = 64;
    static constexpr uint32_t KEY_TILE = 64u * DK * 2u;      // one key tensor, one chunk
    static constexpr uint32_t VAL_TILE = 64u * NV * 2u;      // one value tensor, one chunk
    static constexpr uint32_t CHUNK_BYTES = 4u * KEY_TILE + 2u * VAL_TILE;
    static constexpr uint32_t OFF_Q = 0;
    static constexpr uint32_t OFF_K = OFF_Q + KEY_TILE;
    static constexpr uint32_t OFF_LA = OFF_K + KEY_TILE;
    static constexpr uint32_t OFF_B = OFF_LA + KEY_TILE;
    static constexpr uint32_t OFF_V = OFF_B + KEY_TILE;       // becomes W.V
    static constexpr uint32_t OFF_W = OFF_V + VAL_TILE;
    static constexpr uint32_t OFF_KT = OFF_W + VAL_TILE;      // K~^T  [128 c][64 i]
    static constexpr uint32_t OFF_QE = OFF_KT + 16384;        // Q~^T [128 c][64 r] | E^T/(TE)^T
    static constexpr uint32_t OFF_TP = OFF_QE + 32768;        // [P; T] [128 m][64 i]
    static constexpr uint32_t OFF_S = OFF_TP + 16384;         // bf16 S: NV/64 x [128 c][64 j]
    static constexpr uint32_t OFF_U = OFF_S + (NV / 64) * 16384u;   // U: NV/64 x [64 i][64 j]
    static constexpr uint32_t OFF_GC = OFF_U + (NV / 64) * 8192u;
    static constexpr uint32_t OFF_BAR = OFF_GC + 512;
    static constexpr uint32_t OFF_TMEMP = OFF_BAR + 64;
    static constexpr uint32_t END_MAIN = OFF_TMEMP + 64;
    // fp32 solve scratch: A/T [64][68] + W [16][48]; lives in the log_alpha
    // and b staging tiles (free after prep) when they are large enough.
    static constexpr int LA_STRIDE = 68;
    static constexpr uint32_t SCR_BYTES = (64 * LA_STRIDE + 16 * 48) * 4;
    static constexpr bool SCR_IN_STAGING = 2u * KEY_TILE >= SCR_BYTES;
    static constexpr uint32_t OFF_SCR = SCR_IN_STAGING ? OFF_LA : ((END_MAIN + 1023u) & ~1023u);
    static constexpr uint32_t SMEM_BYTES = SCR_IN_STAGING ? END_MAIN : OFF_SCR + SCR_BYTES;
    static constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;
    // TMEM columns: [AP/ET 64][UT NV][X NV][S NV]
    static constexpr uint32_t T_AP = 0, T_UT = 64, T_X = 64 + NV, T_S = 64 + 2 * NV;
    static constexpr uint32_t TMEM_COLS = (64 + 3 * NV) <= 256 ? 256 : 512;
    static constexpr int PREFETCH = 3;
};

template <int DK, int NV>
__global__ void __launch_bounds__(128, 1)
chunk_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_la, const __grid_constant__ CUtensorMap tm_b,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_w,
                    const float *__restrict__ S0, __nv_bfloat16 *__restrict__ o, float *__restrict__ S_T,
                    int T, int H, int d_v, unsigned long long wait_ns) {
    using Cfg = TcCfg<DK, NV>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(smem);

    const int tid = threadIdx.x, warp = tid >> 5;
    const int j0 = blockIdx.x * NV, h = blockIdx.y, bb = blockIdx.z;
    const int NC = T / Cfg::C;
    const long head = (long)bb * H + h;
    const int row0 = bb * T;   // TMA row coordinate of token 0 of this batch row

    uint64_t *bar_load = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
    uint64_t *bar_mma = bar_load + 1;
    uint64_t *bar_drain = bar_load + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + Cfg::OFF_TMEMP);
    float *gC = reinterpret_cast<float *>(smem + Cfg::OFF_GC);
    float *sA = reinterpret_cast<float *>(smem + Cfg::OFF_SCR);
    float *sW = sA + 64 * Cfg::LA_STRIDE;

    // ---------------------------------------------------------------- setup
    for (uint32_t off = Cfg::OFF_KT + tid * 16u; off < Cfg::OFF_GC; off += 128u * 16u)
        st_shared_v4(sb + off, 0u, 0u, 0u, 0u);
    if (tid == 0) {
        mbar_init(bar_load, 1);
        mbar_init(bar_mma, 1);
        mbar_init(bar_drain, 1);
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
    const uint32_t lane_q = static_cast<uint32_t>(warp * 32) << 16;   // this warp's TMEM lanes
    const uint32_t t_AP = tmem + Cfg::T_AP, t_UT = tmem + Cfg::T_UT;
    const uint32_t t_X = tmem + Cfg::T_X, t_S = tmem + Cfg::T_S;

    auto load_key = [&](const CUtensorMap *m, uint32_t off, int n) {
        for (int kb = 0; kb < DK / 64; ++kb)
            tma_load_3d(smem + off + kb * 8192, m, bar_load, kb * 64, h, row0 + n * 64);
    };
    auto load_val = [&](const CUtensorMap *m, uint32_t off, int n) {
        for (int vb = 0; vb < NV / 64; ++vb)
            tma_load_3d(smem + off + vb * 8192, m, bar_load, j0 + vb * 64, h, row0 + n * 64);
    };
    auto prefetch = [&](int n) {
        const int r = row0 + n * 64;
        for (int kb = 0; kb < DK / 64; ++kb) {
            tma_prefetch_l2_3d(&tm_q, kb * 64, h, r);
            tma_prefetch_l2_3d(&tm_k, kb * 64, h, r);
            tma_prefetch_l2_3d(&tm_la, kb * 64, h, r);
            tma_prefetch_l2_3d(&tm_b, kb * 64, h, r);
        }
        for (int vb = 0; vb < NV / 64; ++vb) {
            tma_prefetch_l2_3d(&tm_v, j0 + vb * 64, h, r);
            tma_prefetch_l2_3d(&tm_w, j0 + vb * 64, h, r);
        }
    };

    if (tid == 0 && NC > 0) {
        mbar_arrive_expect_tx(bar_load, Cfg::CHUNK_BYTES);
        load_key(&tm_la, Cfg::OFF_LA, 0);
        load_key(&tm_q, Cfg::OFF_Q, 0);
        load_key(&tm_k, Cfg::OFF_K, 0);
        load_key(&tm_b, Cfg::OFF_B, 0);
        load_val(&tm_v, Cfg::OFF_V, 0);
        load_val(&tm_w, Cfg::OFF_W, 0);
        for (int p = 1; p <= Cfg::PREFETCH && p < NC; ++p) prefetch(p);
    }

    // initial state: fp32 into TMEM (lane c = key channel), bf16 copy for MMA_s
    {
        const int c = tid;
        for (int jc = 0; jc < NV / 32; ++jc) {
            float s[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) s[e] = 0.f;
            if (S0 != nullptr && c < DK) {
                const float4 *src = reinterpret_cast<const float4 *>(S0 + (head * DK + c) * d_v + j0 + jc * 32);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float4 x = src[e];
                    s[4 * e] = x.x; s[4 * e + 1] = x.y; s[4 * e + 2] = x.z; s[4 * e + 3] = x.w;
                }
            }
            tmem_st32(t_S + lane_q + jc * 32, s);
            const uint32_t tile = sb + Cfg::OFF_S + ((jc * 32) >> 6) * 16384u;
            const uint32_t ch0 = ((jc * 32) & 63) >> 3;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
                st_shared_v4(tile + sw128_chunk(c, ch0 + q4), pack_bf16x2(s[8 * q4], s[8 * q4 + 1]),
                             pack_bf16x2(s[8 * q4 + 2], s[8 * q4 + 3]), pack_bf16x2(s[8 * q4 + 4], s[8 * q4 + 5]),
                             pack_bf16x2(s[8 * q4 + 6], s[8 * q4 + 7]));
        }
    }
    tmem_st_wait();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    uint32_t mma_parity = 0;
    bool failed = false;
    for (int n = 0; n < NC; ++n) {
        // ------------------------------------------------------------ prep
        {
            const bool ok = mbar_wait(bar_load, static_cast<uint32_t>(n & 1), wait_ns);
            if (__syncthreads_or(!ok)) { failed = true; break; }
        }
        {
            const int c = tid;
            if (c < DK) {
                const uint32_t kb = static_cast<uint32_t>(c) >> 6, cc = static_cast<uint32_t>(c) & 63u;
                const uint32_t aq = sb + Cfg::OFF_Q + kb * 8192, ak = sb + Cfg::OFF_K + kb * 8192;
                const uint32_t al = sb + Cfg::OFF_LA + kb * 8192, ab = sb + Cfg::OFF_B + kb * 8192;
                float g = 0.f;
#pragma unroll 1
                for (int rg = 0; rg < 8; ++rg) {
                    uint32_t pq[4], pe[4], pk[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float qv[2], ev[2], kv[2];
#pragma unroll
                        for (int s = 0; s < 2; ++s) {
                            const uint32_t r = rg * 8 + e * 2 + s;
                            const uint32_t off = sw128_off(r, cc);
                            g += ld_shared_bf16(al + off);
                            const float gam = __expf(g), inv = __expf(-g);
                            const float kk = ld_shared_bf16(ak + off);
                            qv[s] = ld_shared_bf16(aq + off) * gam;
                            ev[s] = ld_shared_bf16(ab + off) * kk * gam;
                            kv[s] = kk * inv;
                        }
                        pq[e] = pack_bf16x2(qv[0], qv[1]);
                        pe[e] = pack_bf16x2(ev[0], ev[1]);
                        pk[e] = pack_bf16x2(kv[0], kv[1]);
                    }
                    st_shared_v4(sb + Cfg::OFF_QE + sw128_chunk(c, rg), pq[0], pq[1], pq[2], pq[3]);
                    st_shared_v4(sb + Cfg::OFF_QE + 16384 + sw128_chunk(c, rg), pe[0], pe[1], pe[2], pe[3]);
                    st_shared_v4(sb + Cfg::OFF_KT + sw128_chunk(c, rg), pk[0], pk[1], pk[2], pk[3]);
                }
                gC[c] = __expf(g);
            } else {
                gC[c] = 1.f;
            }
            // W.V in place in the v tile (same layout for v and w)
            for (uint32_t i = tid; i < Cfg::VAL_TILE / 16; i += 128) {
                uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
                ld_shared_v4(sb + Cfg::OFF_V + i * 16, a0, a1, a2, a3);
                ld_shared_v4(sb + Cfg::OFF_W + i * 16, b0, b1, b2, b3);
                st_shared_v4(sb + Cfg::OFF_V + i * 16, pack_bf16x2(bf16_lo(a0) * bf16_lo(b0), bf16_hi(a0) * bf16_hi(b0)),
                             pack_bf16x2(bf16_lo(a1) * bf16_lo(b1), bf16_hi(a1) * bf16_hi(b1)),
                             pack_bf16x2(bf16_lo(a2) * bf16_lo(b2), bf16_hi(a2) * bf16_hi(b2)),
                             pack_bf16x2(bf16_lo(a3) * bf16_lo(b3), bf16_hi(a3) * bf16_hi(b3)));
            }
        }
        fence_proxy_async_smem();
        __syncthreads();
        const bool more = (n + 1 < NC);
        if (tid == 0) {
            if (more) {
                mbar_arrive_expect_tx(bar_load, Cfg::CHUNK_BYTES);
                load_key(&tm_q, Cfg::OFF_Q, n + 1);
                load_key(&tm_k, Cfg::OFF_K, n + 1);
                load_val(&tm_w, Cfg::OFF_W, n + 1);
            }
            if (n + 1 + Cfg::PREFETCH < NC) prefetch(n + 1 + Cfg::PREFETCH);
            // MMA1: [Q~; E] K~^T -> AP
            tc_fence_after();
            const uint32_t id1 = idesc_bf16(128, 64, true, true);
#pragma unroll
            for (int ks = 0; ks < DK / 16; ++ks)
                umma_bf16(t_AP, sdesc_sw128(sb + Cfg::OFF_QE + ks * 2048, 16384, 1024),
                          sdesc_sw128(sb + Cfg::OFF_KT + ks * 2048, 8192, 1024), id1, ks > 0 ? 1u : 0u);
            umma_commit(bar_mma);
        }
        {
            const bool ok = mbar_wait(bar_mma, mma_parity, wait_ns);
            mma_parity ^= 1u;
            if (__syncthreads_or(!ok)) { failed = true; break; }
        }
        tc_fence_after();
        // ------------------------------------------- read out P' and A
        if (warp < 2) {
            const int r = tid;                       // P' row (lanes 0-63)
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
                    st_shared_v4(sb + Cfg::OFF_TP + sw128_chunk(r, half * 4 + q4), p[0], p[1], p[2], p[3]);
                }
            }
        } else {
            const int r = tid - 64;                  // A row (lanes 64-127)
            float *arow = sA + r * Cfg::LA_STRIDE;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float x[32];
                tmem_ld32(t_AP + lane_q + half * 32, x);
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    const int i = half * 32 + e;
                    float4 a;
                    a.x = (i < r) ? x[e] : 0.f;
                    a.y = (i + 1 < r) ? x[e + 1] : 0.f;
                    a.z = (i + 2 < r) ? x[e + 2] : 0.f;
                    a.w = (i + 3 < r) ? x[e + 3] : 0.f;
                    *reinterpret_cast<float4 *>(arow + i) = a;
                }
            }
        }
        __syncthreads();
        // ------------------------------------------ T = (I + A)^{-1}
        // 16x16 diagonal blocks by forward substitution (one column per thread)
        float xd[16];
        const int dblk = tid >> 4, dj = tid & 15, dR = dblk * 16;
        if (tid < 64) {
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float s = (r == dj) ? 1.f : 0.f;
#pragma unroll
                for (int i = 0; i < r; ++i) s = fmaf(-sA[(dR + r) * Cfg::LA_STRIDE + dR + i], xd[i], s);
                xd[r] = s;
            }
        }
        __syncthreads();
        if (tid < 64) {
#pragma unroll
            for (int r = 0; r < 16; ++r) sA[(dR + r) * Cfg::LA_STRIDE + dR + dj] = xd[r];
        }
        __syncthreads();
        // block rows 1..3: T_ib,: = -D_ib (sum_{k<ib} A_ib,k T_k,:)
#pragma unroll 1
        for (int ib = 1; ib < 4; ++ib) {
            const int ncol = 16 * ib;
            for (int idx = tid; idx < 16 * ncol; idx += 128) {
                const int r = idx / ncol, col = idx - r * ncol;
                const float *arow = sA + (16 * ib + r) * Cfg::LA_STRIDE;
                float s = 0.f;
                for (int kk = 0; kk < ncol; ++kk) s = fmaf(arow[kk], sA[kk * Cfg::LA_STRIDE + col], s);
                sW[r * 48 + col] = s;
            }
            __syncthreads();
            for (int idx = tid; idx < 16 * ncol; idx += 128) {
                const int r = idx / ncol, col = idx - r * ncol;
                const float *drow = sA + (16 * ib + r) * Cfg::LA_STRIDE + 16 * ib;
                float s = 0.f;
                for (int ss = 0; ss <= r; ++ss) s = fmaf(drow[ss], sW[ss * 48 + col], s);
                sA[(16 * ib + r) * Cfg::LA_STRIDE + col] = -s;
            }
            __syncthreads();
        }
        // T (fp32) -> bf16 rows 64..127 of TP
        for (int idx = tid; idx < 512; idx += 128) {
            const int r = idx >> 3, ch = idx & 7;
            const float *row = sA + r * Cfg::LA_STRIDE + ch * 8;
            st_shared_v4(sb + Cfg::OFF_TP + sw128_chunk(64 + r, ch), pack_bf16x2(row[0], row[1]),
                         pack_bf16x2(row[2], row[3]), pack_bf16x2(row[4], row[5]), pack_bf16x2(row[6], row[7]));
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            if (more) {
                load_key(&tm_la, Cfg::OFF_LA, n + 1);
                load_key(&tm_b, Cfg::OFF_B, n + 1);
            }
            tc_fence_after();
            // MMA2: (T E)^T = E^T T^T -> AP columns ; MMA3: [P; T] (W.V) -> UT
            const uint32_t id2 = idesc_bf16(128, 64, false, false);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                umma_bf16(t_AP, sdesc_sw128(sb + Cfg::OFF_QE + 16384 + ks * 32, 16, 1024),
                          sdesc_sw128(sb + Cfg::OFF_TP + 8192 + ks * 32, 16, 1024), id2, ks > 0 ? 1u : 0u);
            const uint32_t id3 = idesc_bf16(128, NV, false, true);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                umma_bf16(t_UT, sdesc_sw128(sb + Cfg::OFF_TP + ks * 32, 16, 1024),
                          sdesc_sw128(sb + Cfg::OFF_V + ks * 2048, 8192, 1024), id3, ks > 0 ? 1u : 0u);
            umma_commit(bar_mma);
        }
        {
            const bool ok = mbar_wait(bar_mma, mma_parity, wait_ns);
            mma_parity ^= 1u;
            if (__syncthreads_or(!ok)) { failed = true; break; }
        }
        tc_fence_after();
        if (tid == 0 && more) load_val(&tm_v, Cfg::OFF_V, n + 1);
        // (T E)^T rows c -> bf16 over E^T
        {
            const int c = tid;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float x[32];
                tmem_ld32(t_AP + lane_q + half * 32, x);
                if (c < DK) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        st_shared_v4(sb + Cfg::OFF_QE + 16384 + sw128_chunk(c, half * 4 + q4),
                                     pack_bf16x2(x[8 * q4], x[8 * q4 + 1]), pack_bf16x2(x[8 * q4 + 2], x[8 * q4 + 3]),
                                     pack_bf16x2(x[8 * q4 + 4], x[8 * q4 + 5]), pack_bf16x2(x[8 * q4 + 6], x[8 * q4 + 7]));
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        // ------------------------------------------------------ MMA_s
        if (tid == 0) {
            tc_fence_after();
            const uint32_t ids = idesc_bf16(128, NV, true, true);
#pragma unroll
            for (int ks = 0; ks < DK / 16; ++ks)
                umma_bf16(t_X, sdesc_sw128(sb + Cfg::OFF_QE + ks * 2048, 16384, 1024),
                          sdesc_sw128(sb + Cfg::OFF_S + ks * 2048, 16384, 1024), ids, ks > 0 ? 1u : 0u);
            umma_commit(bar_mma);
        }
        {
            const bool ok = mbar_wait(bar_mma, mma_parity, wait_ns);
            mma_parity ^= 1u;
            if (__syncthreads_or(!ok)) { failed = true; break; }
        }
        tc_fence_after();
        if (warp >= 2) {
            const int r = tid - 64;                  // U row r (lanes 64-127)
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
        __syncthreads();
        // ---------------------------------------------- MMA_u and MMA_o
        if (tid == 0) {
            tc_fence_after();
            const uint32_t idu = idesc_bf16(128, NV, false, true);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t bu = sdesc_sw128(sb + Cfg::OFF_U + ks * 2048, 8192, 1024);
                umma_bf16(t_S, sdesc_sw128(sb + Cfg::OFF_KT + ks * 32, 16, 1024), bu, idu, 1u);
                umma_bf16(t_X, sdesc_sw128(sb + Cfg::OFF_TP + ks * 32, 16, 1024), bu, idu, 1u);
            }
            umma_commit(bar_mma);
        }
        {
            const bool ok = mbar_wait(bar_mma, mma_parity, wait_ns);
            mma_parity ^= 1u;
            if (__syncthreads_or(!ok)) { failed = true; break; }
        }
        tc_fence_after();
        if (warp < 2) {
            const int r = tid;                       // output row r (lanes 0-63)
            __nv_bfloat16 *orow = o + (((long)row0 + n * 64 + r) * H + h) * (long)d_v + j0;
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
        {
            const int c = tid;
            const float gc = gC[c];
            const bool last = (n + 1 == NC);
#pragma unroll 1
            for (int jc = 0; jc < NV / 32; ++jc) {
                float s[32];
                tmem_ld32(t_S + lane_q + jc * 32, s);
#pragma unroll
                for (int e = 0; e < 32; ++e) s[e] *= gc;
                tmem_st32(t_S + lane_q + jc * 32, s);
                if (c < DK) {
                    const uint32_t tile = sb + Cfg::OFF_S + ((jc * 32) >> 6) * 16384u;
                    const uint32_t ch0 = ((jc * 32) & 63) >> 3;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const int e = 8 * q4;
                        st_shared_v4(tile + sw128_chunk(c, ch0 + q4), pack_bf16x2(s[e], s[e + 1]),
                                     pack_bf16x2(s[e + 2], s[e + 3]), pack_bf16x2(s[e + 4], s[e + 5]),
                                     pack_bf16x2(s[e + 6], s[e + 7]));
                    }
                    if (last && S_T != nullptr) {
                        float4 *dst = reinterpret_cast<float4 *>(S_T + (head * DK + c) * d_v + j0 + jc * 32);
#pragma unroll
                        for (int e = 0; e < 8; ++e) dst[e] = make_float4(s[4 * e], s[4 * e + 1], s[4 * e + 2], s[4 * e + 3]);
                    }
                }
            }
        }
        tmem_st_wait();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
    }

    // ------------------------------------------------------------- teardown
    if (failed && tid == 0) {
        record_timeout();
        umma_commit(bar_drain);                 // wait (bounded) for issued MMAs
        mbar_wait(bar_drain, 0u, wait_ns);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, Cfg::TMEM_COLS);
    }
}

}  // namespace gdn2
