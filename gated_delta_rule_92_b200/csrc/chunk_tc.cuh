// chunk_tc.cuh -- chunk-parallel GDN-2 forward on sm_100a tensor cores.
//
// Chunk algebra (the burn-gdn2 README recurrence, "Architecture" section,
// regrouped over chunks of C = 64 tokens as in its "Chunk WY (train)" mode):
//     G = L log_alpha            (L = lower-triangular ones: per-channel cumsum)
//     Q~ = Q.exp(G), K~ = K.exp(-G), E = B.K.exp(G)
//     A = strict_lower(E K~^T),  P = lower(Q~ K~^T),  T = (I + A)^{-1}
//     U = T (W.V) - (T E) S,     O = Q~ S + P U,      S' = diag(exp(G_C)) (S + K~^T U)
// with S the fp32 state at the chunk start.  The README credits its chunk
// speed-up to computing the cumulative sum as a batched matmul; here that is
// one pair of tensor-core MMAs per chunk.
//
// One CTA (13 warps) owns one (b, h, NV-column slice of d_v) and walks the
// T/64 chunks in order as a pipeline:
//   producer warp 12 TMA loads (128B swizzle) of q, k, b (double buffered),
//                   log_alpha, w and v (single buffered), L2 prefetch ahead.
//   key warps 0-7   chunk m, everything that does not depend on the state:
//       MMA_G  G = L log_alpha -> TMEM (two M=64 MMAs: channels 0-63 in the
//              lower half-lanes, 64-127 in the upper half-lanes, so one
//              warp-wide TMEM load hands every thread one row x 64 channels)
//       prep   Q~, E, K~ computed in place in the TMA tiles; W.V in place in
//              the v tile; exp(G_C) for the state update
//       MMA1   [Q~; E] K~^T -> TMEM (rows 0-63 P', rows 64-127 A')
//       solve  T = (I + A)^{-1} in fp32 on CUDA cores (16x16 diagonal blocks
//              by forward substitution, off-diagonal blocks by block products)
//       MMA2   [. ; T] E       -> rows 64-127 = T E, back to bf16 over E
//       MMA3   [. ; T] (W.V)   -> rows 64-127 = T (W.V)
//   chain warps 8-11 chunk m-1, the sequential state pass:
//       MMA_s  [Q~; T E] S -> X (rows 0-63 Q~ S, rows 64-127 T E S)
//       U      = T (W.V) - T E S  (bf16 into shared memory)
//       MMA_u  S += K~^T U   (the fp32 state stays in TMEM across chunks)
//       MMA_o  X += [P; .] U (rows 0-63: O = Q~ S + P U)
//       out    S rows *= exp(G_C) (+ bf16 copy for the next MMA_s); O -> HBM
// All MMAs are tcgen05.mma kind::f16 (bf16 x bf16 -> fp32).  The key and chain
// warpgroups each issue their own MMAs from one thread and track them with
// tcgen05.commit; hand-offs go through mbarriers.  Every wait is bounded; a
// timeout records an error, drains this CTA's MMAs and returns.
#pragma once
#include "gdn2_device.cuh"

namespace gdn2 {

template <int DK, int NV>
struct TcCfg {
    static_assert(DK == 64 || DK == 128, "d_k");
    static_assert(NV == 64 || NV == 128, "value slice");
    static constexpr int C = 64;
    static constexpr int VB = NV / 64;
    static constexpr uint32_t KEY_TILE = 64u * DK * 2u;   // one key tensor, one chunk (TMA bytes)
    static constexpr uint32_t VAL_TILE = 64u * NV * 2u;
    // Stage s holds [Q kb0 | E kb0 | Q kb1 | E kb1] (8 KB blocks of 64 rows x
    // 64 channels), so [Q; E] is a 128-row K-major operand per channel block.
    static constexpr uint32_t OFF_QE0 = 0;
    static constexpr uint32_t OFF_QE1 = 32768;
    static constexpr uint32_t OFF_K0 = 65536;              // K tile [kb][64 i][64 c]
    static constexpr uint32_t OFF_K1 = 81920;
    static constexpr uint32_t OFF_LA = 98304;              // log_alpha [kb][64 s][64 c]; solve scratch
    static constexpr uint32_t OFF_T = OFF_LA + 16384;      // T [64 r][64 i]; its first KB also scratch
    static constexpr uint32_t OFF_W = OFF_T + 8192;        // w [jb][64 i][64 j]
    static constexpr uint32_t OFF_V = OFF_W + VB * 8192u;  // v -> W.V
    static constexpr uint32_t OFF_P0 = OFF_V + VB * 8192u; // P [64 r][64 i], stage 0
    static constexpr uint32_t OFF_P1 = OFF_P0 + 8192;      // P, stage 1
    static constexpr uint32_t OFF_S = OFF_P1 + 8192;       // bf16 S [jb][128 c][64 j]
    static constexpr uint32_t OFF_U = OFF_S + VB * 16384u; // U [jb][64 i][64 j]
    static constexpr uint32_t OFF_L = OFF_U + VB * 8192u;  // L [64 r][64 s]
    static constexpr uint32_t OFF_GC = OFF_L + 8192;       // exp(G_C) [2][128]
    static constexpr uint32_t OFF_BAR = OFF_GC + 1024;
    static constexpr uint32_t OFF_TMEMP = OFF_BAR + 256;
    static constexpr uint32_t SMEM_BYTES = OFF_TMEMP + 16;
    static constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;
    // fp32 solve scratch A/T [64][68], in the log_alpha tile (dead once MMA_G
    // has run) and the first KB of the T tile (rewritten after the solve)
    static constexpr int LDA = 68;
    static constexpr uint32_t OFF_SCR = OFF_LA;
    static_assert(64 * LDA * 4 <= 16384 + 8192, "solve scratch");
    // TMEM columns: [KT 128: G, then P'/A', then T E][T(W.V) NV][X NV][S NV]
    static constexpr uint32_t T_KT = 0, T_UT = 128, T_X = 128 + NV, T_S = 128 + 2 * NV;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr int PREFETCH = 3;
};

// Named barrier over `n` threads (a multiple of 32).
__device__ __forceinline__ void named_bar(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// Named barrier over `n` threads that also ORs a predicate across them.
__device__ __forceinline__ bool group_any(int id, int n, bool p) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.or.pred po, %2, %3, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(p)), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}
constexpr int kKeyThreads = 256;     // warps 0-7
constexpr int kChainThreads = 128;   // warps 8-11
constexpr int kTcThreads = kKeyThreads + kChainThreads + 32;   // + producer warp 12

// T = (I + A)^{-1} for a strictly lower 64x64 A held in fp32 in sA (row
// stride LDA), in place, by the 256 key threads:
//   1. each 16x16 diagonal block D_k = (I + A_kk)^{-1} by right-looking
//      forward substitution, one column per thread (threads 0-63);
//   2. 16 -> 32: T_{2p+1,2p} = -D_{2p+1} (A_{2p+1,2p} D_{2p}), p = 0, 1
//      (threads 0-63);
//   3. 32 -> 64: T_ba = -T_b (A_ba T_a) with a = rows/cols 0-31, b = 32-63
//      (threads 0-127).
// Block products keep two rows of the left factor in registers per thread
// and stream one float4 of the right factor per step, so each 128-bit
// shared-memory load feeds eight FMAs.
// The intermediate products go to the upper-right 32x32 block, which T
// leaves zero; readers of T must mask columns above the diagonal.
// Barriers are named barrier 1 (256 threads).
template <int LDA>
__device__ __forceinline__ void unit_lower_inverse64(float *sA, int t) {
    {   // 1. diagonal blocks
        float x[16];
        const int R = (t >> 4) * 16, j = t & 15;
        if (t < 64) {
            const float *blk = sA + R * LDA + R;
            float sacc[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) sacc[r] = (r == j) ? 1.f : 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                x[i] = sacc[i];
#pragma unroll
                for (int r = i + 1; r < 16; ++r) sacc[r] = fmaf(-blk[r * LDA + i], x[i], sacc[r]);
            }
        }
        named_bar(1, kKeyThreads);
        if (t < 64) {
#pragma unroll
            for (int r = 0; r < 16; ++r) sA[(R + r) * LDA + R + j] = x[r];
        }
        named_bar(1, kKeyThreads);
    }
    {   // 2. 16 -> 32 (threads 0-63: two rows x one float4 each); products in the
        //    upper-right block, rows 16p + r, cols 32 + 4c4
        const int p = (t >> 5) & 1, r = 2 * ((t >> 2) & 7), c4 = t & 3;
        const int R = 32 * p;   // block (2p+1, 2p) lives at rows R+16.., cols R..
        if (t < 64) {
            float a0[16], a1[16];   // rows r, r+1 of A_{2p+1,2p}
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 v0 = *reinterpret_cast<const float4 *>(sA + (R + 16 + r) * LDA + R + 4 * q);
                const float4 v1 = *reinterpret_cast<const float4 *>(sA + (R + 17 + r) * LDA + R + 4 * q);
                a0[4 * q] = v0.x; a0[4 * q + 1] = v0.y; a0[4 * q + 2] = v0.z; a0[4 * q + 3] = v0.w;
                a1[4 * q] = v1.x; a1[4 * q + 1] = v1.y; a1[4 * q + 2] = v1.z; a1[4 * q + 3] = v1.w;
            }
            const float *dcol = sA + R * LDA + R + 4 * c4;
            float4 y0 = make_float4(0.f, 0.f, 0.f, 0.f), y1 = y0;
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const float4 d = *reinterpret_cast<const float4 *>(dcol + k * LDA);
                y0.x = fmaf(a0[k], d.x, y0.x); y0.y = fmaf(a0[k], d.y, y0.y);
                y0.z = fmaf(a0[k], d.z, y0.z); y0.w = fmaf(a0[k], d.w, y0.w);
                y1.x = fmaf(a1[k], d.x, y1.x); y1.y = fmaf(a1[k], d.y, y1.y);
                y1.z = fmaf(a1[k], d.z, y1.z); y1.w = fmaf(a1[k], d.w, y1.w);
            }
            *reinterpret_cast<float4 *>(sA + (16 * p + r) * LDA + 32 + 4 * c4) = y0;
            *reinterpret_cast<float4 *>(sA + (16 * p + r + 1) * LDA + 32 + 4 * c4) = y1;
        }
        named_bar(1, kKeyThreads);
        if (t < 64) {
            float d0[16], d1[16];   // rows r, r+1 of D_{2p+1}
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 v0 = *reinterpret_cast<const float4 *>(sA + (R + 16 + r) * LDA + R + 16 + 4 * q);
                const float4 v1 = *reinterpret_cast<const float4 *>(sA + (R + 17 + r) * LDA + R + 16 + 4 * q);
                d0[4 * q] = v0.x; d0[4 * q + 1] = v0.y; d0[4 * q + 2] = v0.z; d0[4 * q + 3] = v0.w;
                d1[4 * q] = v1.x; d1[4 * q + 1] = v1.y; d1[4 * q + 2] = v1.z; d1[4 * q + 3] = v1.w;
            }
            const float *ycol = sA + (16 * p) * LDA + 32 + 4 * c4;
            float4 z0 = make_float4(0.f, 0.f, 0.f, 0.f), z1 = z0;
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const float4 y = *reinterpret_cast<const float4 *>(ycol + k * LDA);
                z0.x = fmaf(d0[k], y.x, z0.x); z0.y = fmaf(d0[k], y.y, z0.y);
                z0.z = fmaf(d0[k], y.z, z0.z); z0.w = fmaf(d0[k], y.w, z0.w);
                z1.x = fmaf(d1[k], y.x, z1.x); z1.y = fmaf(d1[k], y.y, z1.y);
                z1.z = fmaf(d1[k], y.z, z1.z); z1.w = fmaf(d1[k], y.w, z1.w);
            }
            *reinterpret_cast<float4 *>(sA + (R + 16 + r) * LDA + R + 4 * c4) = make_float4(-z0.x, -z0.y, -z0.z, -z0.w);
            *reinterpret_cast<float4 *>(sA + (R + 17 + r) * LDA + R + 4 * c4) = make_float4(-z1.x, -z1.y, -z1.z, -z1.w);
        }
        named_bar(1, kKeyThreads);
    }
    {   // 3. 32 -> 64 (threads 0-127: two rows x one float4 each); Y in the
        //    upper-right block, rows r, cols 32 + 4c4
        const int r = 2 * (t >> 3), c4 = t & 7;
        if (t < 128) {
            float a0[32], a1[32];   // rows r, r+1 of A_ba
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 v0 = *reinterpret_cast<const float4 *>(sA + (32 + r) * LDA + 4 * q);
                const float4 v1 = *reinterpret_cast<const float4 *>(sA + (33 + r) * LDA + 4 * q);
                a0[4 * q] = v0.x; a0[4 * q + 1] = v0.y; a0[4 * q + 2] = v0.z; a0[4 * q + 3] = v0.w;
                a1[4 * q] = v1.x; a1[4 * q + 1] = v1.y; a1[4 * q + 2] = v1.z; a1[4 * q + 3] = v1.w;
            }
            const float *tcol = sA + 4 * c4;
            float4 y0 = make_float4(0.f, 0.f, 0.f, 0.f), y1 = y0;
#pragma unroll
            for (int k = 0; k < 32; ++k) {   // Y = A_ba T_a
                const float4 tv = *reinterpret_cast<const float4 *>(tcol + k * LDA);
                y0.x = fmaf(a0[k], tv.x, y0.x); y0.y = fmaf(a0[k], tv.y, y0.y);
                y0.z = fmaf(a0[k], tv.z, y0.z); y0.w = fmaf(a0[k], tv.w, y0.w);
                y1.x = fmaf(a1[k], tv.x, y1.x); y1.y = fmaf(a1[k], tv.y, y1.y);
                y1.z = fmaf(a1[k], tv.z, y1.z); y1.w = fmaf(a1[k], tv.w, y1.w);
            }
            *reinterpret_cast<float4 *>(sA + r * LDA + 32 + 4 * c4) = y0;
            *reinterpret_cast<float4 *>(sA + (r + 1) * LDA + 32 + 4 * c4) = y1;
        }
        named_bar(1, kKeyThreads);
        if (t < 128) {
            float d0[32], d1[32];   // rows r, r+1 of T_b (zero above the diagonal)
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 v0 = *reinterpret_cast<const float4 *>(sA + (32 + r) * LDA + 32 + 4 * q);
                const float4 v1 = *reinterpret_cast<const float4 *>(sA + (33 + r) * LDA + 32 + 4 * q);
                d0[4 * q] = v0.x; d0[4 * q + 1] = v0.y; d0[4 * q + 2] = v0.z; d0[4 * q + 3] = v0.w;
                d1[4 * q] = v1.x; d1[4 * q + 1] = v1.y; d1[4 * q + 2] = v1.z; d1[4 * q + 3] = v1.w;
            }
            const float *ycol = sA + 32 + 4 * c4;
            float4 z0 = make_float4(0.f, 0.f, 0.f, 0.f), z1 = z0;
#pragma unroll
            for (int k = 0; k < 32; ++k) {   // T_ba = -T_b Y
                const float4 y = *reinterpret_cast<const float4 *>(ycol + k * LDA);
                z0.x = fmaf(d0[k], y.x, z0.x); z0.y = fmaf(d0[k], y.y, z0.y);
                z0.z = fmaf(d0[k], y.z, z0.z); z0.w = fmaf(d0[k], y.w, z0.w);
                z1.x = fmaf(d1[k], y.x, z1.x); z1.y = fmaf(d1[k], y.y, z1.y);
                z1.z = fmaf(d1[k], y.z, z1.z); z1.w = fmaf(d1[k], y.w, z1.w);
            }
            *reinterpret_cast<float4 *>(sA + (32 + r) * LDA + 4 * c4) = make_float4(-z0.x, -z0.y, -z0.z, -z0.w);
            *reinterpret_cast<float4 *>(sA + (33 + r) * LDA + 4 * c4) = make_float4(-z1.x, -z1.y, -z1.z, -z1.w);
        }
        named_bar(1, kKeyThreads);
    }
}

// 8 bf16 products of two 16-byte vectors, rounded back to bf16.
__device__ __forceinline__ uint4 mul_bf16x8(const uint4 &a, const uint4 &b) {
    return make_uint4(pack_bf16x2(bf16_lo(a.x) * bf16_lo(b.x), bf16_hi(a.x) * bf16_hi(b.x)),
                      pack_bf16x2(bf16_lo(a.y) * bf16_lo(b.y), bf16_hi(a.y) * bf16_hi(b.y)),
                      pack_bf16x2(bf16_lo(a.z) * bf16_lo(b.z), bf16_hi(a.z) * bf16_hi(b.z)),
                      pack_bf16x2(bf16_lo(a.w) * bf16_lo(b.w), bf16_hi(a.w) * bf16_hi(b.w)));
}

template <int DK, int NV>
__global__ void __launch_bounds__(kTcThreads, 1)
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
    const int NC = (T + Cfg::C - 1) / Cfg::C;   // the last chunk may be partial
    const long head = (long)bb * H + h;

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
    uint64_t *qkb_full = bars + 0;    // [2] TMA q, k, b of a chunk landed (stage)
    uint64_t *lw_full = bars + 2;     // TMA log_alpha, w landed
    uint64_t *v_full = bars + 3;      // TMA v landed
    uint64_t *lw_free = bars + 4;     // key done with log_alpha/w tiles (and the solve scratch)
    uint64_t *v_free = bars + 5;      // key done with W.V (MMA3 complete)
    uint64_t *full = bars + 6;        // [2] key products of a chunk ready
    uint64_t *empty = bars + 8;       // [2] chain done with a stage
    uint64_t *utfree = bars + 10;     // chain read T(W.V) and MMA_s done
    uint64_t *bG = bars + 11, *bk1 = bars + 12, *bk2 = bars + 13;
    uint64_t *bc1 = bars + 14, *bc2 = bars + 15, *bc3 = bars + 16;
    uint64_t *drain = bars + 17;      // [2]
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + Cfg::OFF_TMEMP);
    float *gC = reinterpret_cast<float *>(smem + Cfg::OFF_GC);
    float *sA = reinterpret_cast<float *>(smem + Cfg::OFF_SCR);

    // ---------------------------------------------------------------- setup
    for (uint32_t off = tid * 16u; off < Cfg::OFF_L; off += kTcThreads * 16u) st_shared_v4(sb + off, 0u, 0u, 0u, 0u);
    for (int i = tid; i < 512; i += kTcThreads) {   // L: lower-triangular ones, K-major [r][s]
        const int r = i >> 3, ch = i & 7;
        uint32_t p[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int s0 = ch * 8 + 2 * e;
            p[e] = pack_bf16x2(s0 <= r ? 1.f : 0.f, s0 + 1 <= r ? 1.f : 0.f);
        }
        st_shared_v4(sb + Cfg::OFF_L + sw128_chunk(r, ch), p[0], p[1], p[2], p[3]);
    }
    if (tid == 0) {
        for (int i = 0; i < 19; ++i) mbar_init(bars + i, 1);
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
    const uint32_t t_KT = tmem + Cfg::T_KT, t_UT = tmem + Cfg::T_UT;
    const uint32_t t_X = tmem + Cfg::T_X, t_S = tmem + Cfg::T_S;
    bool failed = false;

    if (warp == 12) {
        // ============================================================ producer
        if ((tid & 31) == 0 && NC > 0) {
            // Token tiles are addressed (channel, head, token, batch); rows past T
            // are outside the tensor and TMA fills them with zeros, which makes
            // padded tokens exact no-ops of the recurrence (k = q = b = w = 0 and
            // log_alpha = 0).
            auto prefetch = [&](int n) {
                const int r = n * 64;
                for (int kb = 0; kb < DK / 64; ++kb) {
                    tma_prefetch_l2_4d(&tm_la, kb * 64, h, r, bb);
                    tma_prefetch_l2_4d(&tm_q, kb * 64, h, r, bb);
                    tma_prefetch_l2_4d(&tm_k, kb * 64, h, r, bb);
                    tma_prefetch_l2_4d(&tm_b, kb * 64, h, r, bb);
                }
                for (int vb = 0; vb < Cfg::VB; ++vb) {
                    tma_prefetch_l2_4d(&tm_v, j0 + vb * 64, h, r, bb);
                    tma_prefetch_l2_4d(&tm_w, j0 + vb * 64, h, r, bb);
                }
            };
            for (int p = 0; p < Cfg::PREFETCH && p < NC; ++p) prefetch(p);
            int nq = 0, nl = 0, nv = 0;   // next chunk to load for each group
            uint64_t t0 = globaltimer_ns();
            while (nq < NC || nl < NC || nv < NC) {
                bool progress = false;
                if (nq < NC && (nq < 2 || mbar_try_wait(&empty[nq & 1], static_cast<uint32_t>(((nq >> 1) - 1) & 1)))) {
                    const int s = nq & 1, r = nq * 64;
                    const uint32_t oqe = s ? Cfg::OFF_QE1 : Cfg::OFF_QE0, ok = s ? Cfg::OFF_K1 : Cfg::OFF_K0;
                    mbar_arrive_expect_tx(&qkb_full[s], 3u * Cfg::KEY_TILE);
                    for (int kb = 0; kb < DK / 64; ++kb) {
                        tma_load_4d(smem + oqe + kb * 16384, &tm_q, &qkb_full[s], kb * 64, h, r, bb);
                        tma_load_4d(smem + oqe + kb * 16384 + 8192, &tm_b, &qkb_full[s], kb * 64, h, r, bb);
                        tma_load_4d(smem + ok + kb * 8192, &tm_k, &qkb_full[s], kb * 64, h, r, bb);
                    }
                    if (nq + Cfg::PREFETCH < NC) prefetch(nq + Cfg::PREFETCH);
                    ++nq;
                    progress = true;
                }
                if (nl < NC && nl < nq && (nl < 1 || mbar_try_wait(lw_free, static_cast<uint32_t>((nl - 1) & 1)))) {
                    const int r = nl * 64;
                    mbar_arrive_expect_tx(lw_full, Cfg::KEY_TILE + Cfg::VAL_TILE);
                    for (int kb = 0; kb < DK / 64; ++kb)
                        tma_load_4d(smem + Cfg::OFF_LA + kb * 8192, &tm_la, lw_full, kb * 64, h, r, bb);
                    for (int vb = 0; vb < Cfg::VB; ++vb)
                        tma_load_4d(smem + Cfg::OFF_W + vb * 8192, &tm_w, lw_full, j0 + vb * 64, h, r, bb);
                    ++nl;
                    progress = true;
                }
                if (nv < NC && nv < nq && (nv < 1 || mbar_try_wait(v_free, static_cast<uint32_t>((nv - 1) & 1)))) {
                    const int r = nv * 64;
                    mbar_arrive_expect_tx(v_full, Cfg::VAL_TILE);
                    for (int vb = 0; vb < Cfg::VB; ++vb)
                        tma_load_4d(smem + Cfg::OFF_V + vb * 8192, &tm_v, v_full, j0 + vb * 64, h, r, bb);
                    ++nv;
                    progress = true;
                }
                const uint64_t now = globaltimer_ns();
                if (progress) t0 = now;
                else if (now - t0 > wait_ns) { failed = true; break; }
            }
        }
    } else if (tid < kKeyThreads) {
        // ============================================================ key side
        const int t = tid, l = tid & 31, kq = warp & 3, kh = warp >> 2;   // lane quarter, column half
        const int prow = 16 * kq + (l & 15), phf = l >> 4;   // prep: row, channel half
        uint32_t phG = 0, ph1 = 0, ph2 = 0;
        for (int m = 0; m < NC; ++m) {
            const int s = m & 1;
            const uint32_t OQE = s ? Cfg::OFF_QE1 : Cfg::OFF_QE0, OK = s ? Cfg::OFF_K1 : Cfg::OFF_K0;
            const uint32_t OP = s ? Cfg::OFF_P1 : Cfg::OFF_P0;
            // ------------------------------------------------- MMA_G (cumsum)
            {
                const bool ok = mbar_wait(lw_full, static_cast<uint32_t>(m & 1), wait_ns);
                if (group_any(1, kKeyThreads, !ok)) { failed = true; break; }
            }
            if (t == 0) {
                tc_fence_after();
                const uint32_t idg = idesc_bf16(64, 64, false, true);
                for (int kb = 0; kb < DK / 64; ++kb)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        umma_bf16(t_KT + (static_cast<uint32_t>(16 * kb) << 16), sdesc_sw128(sb + Cfg::OFF_L + ks * 32, 16, 1024),
                                  sdesc_sw128(sb + Cfg::OFF_LA + kb * 8192 + ks * 2048, 8192, 1024), idg,
                                  ks > 0 ? 1u : 0u);
                umma_commit(bG);
            }
            {
                bool ok = mbar_wait(&qkb_full[s], static_cast<uint32_t>((m >> 1) & 1), wait_ns);
                ok = ok && mbar_wait(bG, phG, wait_ns);
                phG ^= 1u;
                if (group_any(1, kKeyThreads, !ok)) { failed = true; break; }
            }
            tc_fence_after();
            // ------------------------------------------------------ prep
            // thread: row prow, channels phf*64 + 32*kh + [0, 32)
            {
                float gv[32];
                tmem_ld32(t_KT + lane_q + 32 * kh, gv);
                if (phf < DK / 64) {
                    const uint32_t qb = sb + OQE + phf * 16384, eb = qb + 8192, kb = sb + OK + phf * 8192;
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const uint32_t co = sw128_chunk(prow, 4 * kh + jj);
                        uint32_t q0, q1, q2, q3, k0, k1, k2, k3, b0, b1, b2, b3;
                        ld_shared_v4(qb + co, q0, q1, q2, q3);
                        ld_shared_v4(kb + co, k0, k1, k2, k3);
                        ld_shared_v4(eb + co, b0, b1, b2, b3);
                        const uint32_t qw[4] = {q0, q1, q2, q3}, kw[4] = {k0, k1, k2, k3}, bw[4] = {b0, b1, b2, b3};
                        uint32_t oq[4], oe[4], okk[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float g0 = gv[8 * jj + 2 * e], g1 = gv[8 * jj + 2 * e + 1];
                            const float ga0 = __expf(g0), ga1 = __expf(g1);
                            const float iv0 = __expf(-g0), iv1 = __expf(-g1);
                            const float kv0 = bf16_lo(kw[e]), kv1 = bf16_hi(kw[e]);
                            oq[e] = pack_bf16x2(bf16_lo(qw[e]) * ga0, bf16_hi(qw[e]) * ga1);
                            oe[e] = pack_bf16x2(bf16_lo(bw[e]) * kv0 * ga0, bf16_hi(bw[e]) * kv1 * ga1);
                            okk[e] = pack_bf16x2(kv0 * iv0, kv1 * iv1);
                        }
                        st_shared_v4(qb + co, oq[0], oq[1], oq[2], oq[3]);
                        st_shared_v4(eb + co, oe[0], oe[1], oe[2], oe[3]);
                        st_shared_v4(kb + co, okk[0], okk[1], okk[2], okk[3]);
                    }
                    if (prow == 63) {
#pragma unroll
                        for (int ch = 0; ch < 32; ++ch) gC[s * 128 + phf * 64 + 32 * kh + ch] = __expf(gv[ch]);
                    }
                } else if (prow == 63) {
                    for (int ch = 0; ch < 32; ++ch) gC[s * 128 + phf * 64 + 32 * kh + ch] = 1.f;
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar(1, kKeyThreads);
            // ---------------------------------------------------------- MMA1
            if (t == 0) {
                tc_fence_after();
                const uint32_t id1 = idesc_bf16(128, 64, false, false);
#pragma unroll
                for (int ks = 0; ks < DK / 16; ++ks)
                    umma_bf16(t_KT, sdesc_sw128(sb + OQE + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
                              sdesc_sw128(sb + OK + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024), id1,
                              ks > 0 ? 1u : 0u);
                umma_commit(bk1);
            }
            // W.V in place in the v tile while MMA1 runs (the solve scratch does not
            // touch the w tile)
            {
                const bool ok = mbar_wait(v_full, static_cast<uint32_t>(m & 1), wait_ns);
                if (group_any(1, kKeyThreads, !ok)) { failed = true; break; }
#pragma unroll
                for (int it = 0; it < Cfg::VAL_TILE / 16 / kKeyThreads; ++it) {
                    const uint32_t off = (t + it * kKeyThreads) * 16u;
                    uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
                    ld_shared_v4(sb + Cfg::OFF_V + off, a0, a1, a2, a3);
                    ld_shared_v4(sb + Cfg::OFF_W + off, b0, b1, b2, b3);
                    const uint4 r4 = mul_bf16x8(make_uint4(a0, a1, a2, a3), make_uint4(b0, b1, b2, b3));
                    st_shared_v4(sb + Cfg::OFF_V + off, r4.x, r4.y, r4.z, r4.w);
                }
            }
            {
                const bool ok = mbar_wait(bk1, ph1, wait_ns);
                ph1 ^= 1u;
                if (group_any(1, kKeyThreads, !ok)) { failed = true; break; }
            }
            tc_fence_after();
            // ------------------------------------------- read out P' and A
            // warp: lanes 32*kq.., columns 32*kh..; P' in lanes 0-63, A' in 64-127
            {
                float x[32];
                tmem_ld32(t_KT + lane_q + 32 * kh, x);
                if (kq < 2) {
                    const int r = 32 * kq + l;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        uint32_t pp[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int i = 32 * kh + q4 * 8 + 2 * e;
                            pp[e] = pack_bf16x2(i <= r ? x[q4 * 8 + 2 * e] : 0.f, i + 1 <= r ? x[q4 * 8 + 2 * e + 1] : 0.f);
                        }
                        st_shared_v4(sb + OP + sw128_chunk(r, 4 * kh + q4), pp[0], pp[1], pp[2], pp[3]);
                    }
                } else {
                    const int r = 32 * (kq - 2) + l;
#pragma unroll
                    for (int e = 0; e < 32; e += 4) {
                        const int i = 32 * kh + e;
                        *reinterpret_cast<float4 *>(sA + r * Cfg::LDA + i) =
                            make_float4(i < r ? x[e] : 0.f, i + 1 < r ? x[e + 1] : 0.f, i + 2 < r ? x[e + 2] : 0.f,
                                        i + 3 < r ? x[e + 3] : 0.f);
                    }
                }
            }
            tc_fence_before();
            named_bar(1, kKeyThreads);
            // ------------------------------------------ T = (I + A)^{-1}
            unit_lower_inverse64<Cfg::LDA>(sA, t);
            {   // T (fp32 scratch) -> bf16 T tile; read everything before writing, since
                // the scratch's last rows overlap the T tile
                uint32_t tp[2][4];
#pragma unroll
                for (int it = 0; it < 2; ++it) {
                    const int idx = t + it * kKeyThreads, r = idx >> 3, ch = idx & 7, c0 = 8 * ch;
                    const float4 a = *reinterpret_cast<const float4 *>(sA + r * Cfg::LDA + c0);
                    const float4 b4 = *reinterpret_cast<const float4 *>(sA + r * Cfg::LDA + c0 + 4);
                    // T is unit lower triangular; the scratch above the diagonal is not T
                    tp[it][0] = pack_bf16x2(c0 <= r ? a.x : 0.f, c0 + 1 <= r ? a.y : 0.f);
                    tp[it][1] = pack_bf16x2(c0 + 2 <= r ? a.z : 0.f, c0 + 3 <= r ? a.w : 0.f);
                    tp[it][2] = pack_bf16x2(c0 + 4 <= r ? b4.x : 0.f, c0 + 5 <= r ? b4.y : 0.f);
                    tp[it][3] = pack_bf16x2(c0 + 6 <= r ? b4.z : 0.f, c0 + 7 <= r ? b4.w : 0.f);
                }
                named_bar(1, kKeyThreads);
#pragma unroll
                for (int it = 0; it < 2; ++it) {
                    const int idx = t + it * kKeyThreads, r = idx >> 3, ch = idx & 7;
                    st_shared_v4(sb + Cfg::OFF_T + sw128_chunk(r, ch), tp[it][0], tp[it][1], tp[it][2], tp[it][3]);
                }
            }
            fence_proxy_async_smem();
            named_bar(1, kKeyThreads);
            if (t == 0) mbar_arrive(lw_free);   // log_alpha (scratch) and w tiles are free
            // the chain must have read T(W.V) and run MMA_s of the previous chunk
            if (m >= 1) {
                const bool ok = mbar_wait(utfree, static_cast<uint32_t>((m - 1) & 1), wait_ns);
                if (group_any(1, kKeyThreads, !ok)) { failed = true; break; }
            }
            // ------------------------------------------------ MMA2 + MMA3
            if (t == 0) {
                tc_fence_after();
                const uint32_t id2 = idesc_bf16(128, DK, false, true);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_bf16(t_KT, sdesc_sw128(sb + Cfg::OFF_T - 8192 + ks * 32, 16, 1024),
                              sdesc_sw128(sb + OQE + 8192 + ks * 2048, 16384, 1024), id2, ks > 0 ? 1u : 0u);
                const uint32_t id3 = idesc_bf16(128, NV, false, true);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_bf16(t_UT, sdesc_sw128(sb + Cfg::OFF_T - 8192 + ks * 32, 16, 1024),
                              sdesc_sw128(sb + Cfg::OFF_V + ks * 2048, 8192, 1024), id3, ks > 0 ? 1u : 0u);
                umma_commit(bk2);
            }
            {
                const bool ok = mbar_wait(bk2, ph2, wait_ns);
                ph2 ^= 1u;
                if (group_any(1, kKeyThreads, !ok)) { failed = true; break; }
            }
            tc_fence_after();
            if (t == 0) mbar_arrive(v_free);
            // T E rows (TMEM lanes 64-127) -> bf16 over E; channel block kb = kh
            if (kq >= 2 && kh < DK / 64) {
                const int r = 32 * (kq - 2) + l;
                const uint32_t eb = sb + OQE + kh * 16384 + 8192;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float x[32];
                    tmem_ld32(t_KT + lane_q + kh * 64 + half * 32, x);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        st_shared_v4(eb + sw128_chunk(r, half * 4 + q4), pack_bf16x2(x[8 * q4], x[8 * q4 + 1]),
                                     pack_bf16x2(x[8 * q4 + 2], x[8 * q4 + 3]), pack_bf16x2(x[8 * q4 + 4], x[8 * q4 + 5]),
                                     pack_bf16x2(x[8 * q4 + 6], x[8 * q4 + 7]));
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar(1, kKeyThreads);
            if (t == 0) mbar_arrive(&full[s]);
        }
        if (t == 0) {   // wait (bounded) for this issuer's MMAs before teardown
            umma_commit(&drain[0]);
            mbar_wait(&drain[0], 0u, wait_ns);
        }
    } else {
        // ========================================================== chain side
        const int t = tid - kKeyThreads;
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
            named_bar(2, kChainThreads);
        }
        uint32_t ph1 = 0, ph2 = 0, ph3 = 0;
        for (int n = 0; n < NC; ++n) {
            const int s = n & 1;
            const uint32_t OQE = s ? Cfg::OFF_QE1 : Cfg::OFF_QE0, OK = s ? Cfg::OFF_K1 : Cfg::OFF_K0;
            const uint32_t OP = s ? Cfg::OFF_P1 : Cfg::OFF_P0;
            {
                const bool ok = mbar_wait(&full[s], static_cast<uint32_t>((n >> 1) & 1), wait_ns);
                if (group_any(2, kChainThreads, !ok)) { failed = true; break; }
            }
            // ------------------------------------------------------ MMA_s
            if (t == 0) {
                tc_fence_after();
                const uint32_t ids = idesc_bf16(128, NV, false, true);
#pragma unroll
                for (int ks = 0; ks < DK / 16; ++ks)
                    umma_bf16(t_X, sdesc_sw128(sb + OQE + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
                              sdesc_sw128(sb + Cfg::OFF_S + ks * 2048, 16384, 1024), ids, ks > 0 ? 1u : 0u);
                umma_commit(bc1);
            }
            {
                const bool ok = mbar_wait(bc1, ph1, wait_ns);
                ph1 ^= 1u;
                if (group_any(2, kChainThreads, !ok)) { failed = true; break; }
            }
            tc_fence_after();
            if ((warp & 3) >= 2) {
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
            named_bar(2, kChainThreads);
            // ---------------------------------------------- MMA_u and MMA_o
            if (t == 0) {
                mbar_arrive(utfree);
                tc_fence_after();
                const uint32_t idu = idesc_bf16(128, NV, true, true);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_bf16(t_S, sdesc_sw128(sb + OK + ks * 2048, 8192, 1024),
                              sdesc_sw128(sb + Cfg::OFF_U + ks * 2048, 8192, 1024), idu, 1u);
                umma_commit(bc2);
                const uint32_t ido = idesc_bf16(128, NV, false, true);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_bf16(t_X, sdesc_sw128(sb + OP + ks * 32, 16, 1024),
                              sdesc_sw128(sb + Cfg::OFF_U + ks * 2048, 8192, 1024), ido, 1u);
                umma_commit(bc3);
            }
            {
                const bool ok = mbar_wait(bc2, ph2, wait_ns);
                ph2 ^= 1u;
                if (group_any(2, kChainThreads, !ok)) { failed = true; break; }
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
                if (group_any(2, kChainThreads, !ok)) { failed = true; break; }
            }
            tc_fence_after();
            if ((warp & 3) < 2) {
                const int r = t;   // output row r (TMEM lanes 0-63); rows past T are padding
                const bool valid = n * 64 + r < T;
                __nv_bfloat16 *orow = o + (((long)bb * T + (long)n * 64 + r) * H + h) * (long)d_v + j0;
#pragma unroll 1
                for (int jc = 0; jc < NV / 32; ++jc) {
                    float x[32];
                    tmem_ld32(t_X + lane_q + jc * 32, x);
                    if (valid) {
                        uint4 *dst = reinterpret_cast<uint4 *>(orow + jc * 32);
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const int e = 8 * q4;
                            dst[q4] = make_uint4(pack_bf16x2(x[e], x[e + 1]), pack_bf16x2(x[e + 2], x[e + 3]),
                                                 pack_bf16x2(x[e + 4], x[e + 5]), pack_bf16x2(x[e + 6], x[e + 7]));
                        }
                    }
                }
            }
            tmem_st_wait();
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar(2, kChainThreads);
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
