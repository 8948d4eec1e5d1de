// chunk_tc.cuh -- chunk-parallel GDN-2 forward on sm_100a tensor cores.
//
// Chunk algebra (the burn-gdn2 README recurrence, "Architecture" section,
// regrouped over chunks of C = 64 tokens as in its "Chunk WY (train)" mode):
//     G = cumsum_rows(log_alpha)  (per key channel),  ref = (G_0 + G_C) / 2
//     Q~ = Q.exp(G - ref), K~ = K.exp(ref - G), E = B.K.exp(G - ref)
//     A = strict_lower(E K~^T),  P = lower(Q~ K~^T),  T = (I + A)^{-1}
//     U = T (W.V) - T (E S_r),   O = Q~ S_r + P U,    S' = diag(exp(G_C - ref)) (S_r + K~^T U)
// with S the fp32 state at the chunk start and S_r = diag(exp(ref)) S the state
// as the chain carries it.  The reference point in the middle of the chunk's
// decay range keeps every operand within exp(+-span / 2), span = G_0 - G_C; a
// chunk whose span passes kMaxChunkSpan2 (log2 units) is not evaluated this way:
// it and the rest of its sequence run token by token (tc_token_tail), so the
// kernel is exact for any decay.
//
// One CTA (13 warps) owns one (b, h, NV-column slice of d_v) and walks the
// T/64 chunks in order as a pipeline:
//   producer warp 12 TMA loads (128B swizzle) of q, b (double buffered), k
//                   (triple buffered), w and v (single buffered, each refilled
//                   as soon as its last reader is done), L2 prefetch ahead;
//                   log_alpha goes straight to the prep threads' registers.
//   key warps 0-7   chunk m, everything that does not depend on the state:
//       prep   G by a running fp32 sum per channel quad, the chunk's span and
//              reference point, then Q~, E, K~ in place in the TMA tiles and
//              exp(G_C - ref), exp(ref) for the state update
//       W.V    in place in the v tile
//       MMA1   [Q~; E] K~^T -> TMEM (rows 0-63 P', rows 64-127 A')
//       solve  T = (I + A)^{-1} in fp32 (16x16 diagonal blocks by forward
//              substitution, off-diagonal blocks by tf32 mma.sync block
//              products), each block of T written to its bf16 MMA tile as soon
//              as it is final
//       MMA3   [. ; T] (W.V)   -> rows 64-127 = T (W.V) in TMEM; its commits
//              free the v tile and hand T (W.V) to the chain
//     as a two-stage pipeline: warps 0-3 solve chunk m while warps 4-7 run
//     the prep of chunk m+1 (the state factors are triple buffered for that)
//   chain warps 8-11 chunk m-1, the sequential state pass:
//       MMA_s  [Q~; E] S -> X (rows 0-63 Q~ S, rows 64-127 E S)
//       -E S   to bf16 over the E tiles
//       MMA_T  [. ; T] (-E S) accumulated onto T (W.V): rows 64-127 = U,
//              bf16 into shared memory
//       MMA_u  S += K~^T U   (the fp32 state stays in TMEM across chunks)
//       MMA_o  X += [P; .] U (rows 0-63: O = Q~ S + P U)
//       out    S rows *= exp(G_C - ref), then *= exp(ref') of the next chunk (+ bf16
//              copy for the next MMA_s); O -> HBM through the U tile and a TMA store
// All MMAs are tcgen05.mma kind::f16 (bf16 x bf16 -> fp32).  The key and chain
// warpgroups each issue their own MMAs from one thread and track them with
// tcgen05.commit; hand-offs go through mbarriers.  Every wait is bounded; a
// timeout records an error, drains this CTA's MMAs and returns.
#pragma once
#include <type_traits>

#include "decode.cuh"
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
    static constexpr uint32_t OFF_K = 65536;               // K tiles [3 stages][kb][64 i][64 c]
    static constexpr uint32_t OFF_W = OFF_K + 3 * 16384;   // w [jb][64 i][64 j] (16 KB reserved); solve scratch
    static constexpr uint32_t OFF_T = OFF_W + 16384 + 1024; // T [64 r][64 i], after the scratch's last KB
    static constexpr uint32_t OFF_V = OFF_T + 8192;        // v -> W.V
    static constexpr uint32_t OFF_P0 = OFF_V + VB * 8192u; // P [64 r][64 i], stage 0
    static constexpr uint32_t OFF_P1 = OFF_P0 + 8192;      // P, stage 1
    static constexpr uint32_t OFF_S = OFF_P1 + 8192;       // bf16 S [jb][128 c][64 j]
    static constexpr uint32_t OFF_U = OFF_S + VB * 16384u; // U [jb][64 i][64 j]
    static constexpr uint32_t OFF_CARRY = OFF_U + VB * 8192u;   // cumsum carries [row block][128], row 0 [128]
    static constexpr uint32_t OFF_GC = OFF_CARRY + 2560;         // state factors [3][2][128]
    static constexpr uint32_t OFF_NRM = OFF_GC + 3072;           // fused prep: 1/|q_r|, 1/|k_r| [64][2]
    static constexpr uint32_t OFF_NW = OFF_NRM + 512;            // fused epilogue: norm weight [NV]
    static constexpr uint32_t OFF_RMS = OFF_NW + 512;            // fused epilogue: 1 / rms(o_r) [64]
    static constexpr uint32_t OFF_BAR = OFF_RMS + 256;
    static constexpr uint32_t OFF_TMEMP = OFF_BAR + 256;   // up to 32 mbarriers
    static constexpr uint32_t OFF_STOP = OFF_TMEMP + 4;    // first chunk handed to the token tail
    static constexpr uint32_t OFF_SEQ = OFF_TMEMP + 8;     // this CTA's sequence: tok0 (8 B), len, bb
    static constexpr uint32_t SMEM_BYTES = OFF_TMEMP + 24;
    static constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;
    static_assert(OFF_T % 1024 == 0 && OFF_V % 1024 == 0 && OFF_S % 1024 == 0 && SMEM_ALLOC <= 232448, "layout");
    // fp32 solve scratch A/T [64][68]: the w tile (dead once W.V is formed) and
    // the KB after it; T itself is read by the chain's MMA_T while the next
    // chunk's A is read out, so it does not overlap the scratch
    static constexpr int LDA = 68;
    static constexpr uint32_t OFF_SCR = OFF_W;
    // -E S of a chunk (64 tokens x NV, two 64-column halves) goes over the E
    // tiles of its Q~/E stage (DK = 64: over Q~ and E)
    __host__ __device__ static constexpr uint32_t es_tile(int half) { return DK == 128 ? 8192u + half * 16384u : half * 8192u; }
    static constexpr uint32_t ES_LBO = DK == 128 ? 16384u : 8192u;
    static_assert(64 * LDA * 4 <= 16384 + 1024, "solve scratch");
    // TMEM columns: [KT 128: P'/A' (64 used)][T(W.V), then U NV][X NV][S NV]
    static constexpr uint32_t T_KT = 0, T_UT = 128, T_X = 128 + NV, T_S = 128 + 2 * NV;
    static constexpr uint32_t TMEM_COLS = 512;
};

// Named barrier over `n` threads (a multiple of 32).
__device__ __forceinline__ void named_bar(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// Arrive on named barrier `id` (of `n` threads) without waiting: the producer
// side of a hand-off whose consumers wait with named_bar(id, n).
__device__ __forceinline__ void named_bar_arrive(int id, int n) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
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
// Largest decay span, in log2 units, that a chunk may have for the tensor-core
// form: over rows 1..63, sum_r log2(alpha_r) >= -kMaxChunkSpan2 in every channel.
// The operands then stay within 2^(+-100): the masked (upper) products may
// overflow and are discarded by selection, every kept product is bounded by
// |q| |k|, and the state update K~^T U stays below 2^128 while |k| |U| < 2^22.
// A chunk past it (a mean decay below about 0.11 per token over the chunk) and
// the rest of its sequence go to the token tail.
constexpr float kMaxChunkSpan2 = 200.f;

constexpr int kKeyThreads = 256;     // warps 0-7
constexpr int kChainThreads = 128;   // warps 8-11
constexpr int kTcThreads = kKeyThreads + kChainThreads + 32;   // + producer warp 12

// fp32 -> tf32 (round to nearest, ties away from zero), as a tensor-core operand.
__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
// D += A B for one m16n8k8 tile (tf32 inputs, fp32 accumulation), warp-wide.
// Fragments (g = lane / 4, q = lane % 4): a = A[g][q], A[g+8][q], A[g][q+4],
// A[g+8][q+4];  b = B[q][g], B[q+4][g];  d = D[g][2q], D[g][2q+1], D[g+8][2q],
// D[g+8][2q+1].
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// One warp: C (16 x 8 NNT, row stride LDA) = sign * Am (16 x K) Bm (K x 8 NNT),
// all in fp32 shared memory with row stride LDA, products in tf32 on the
// tensor cores.  With a tile `tt`, C also goes, rounded to bf16, to rows
// trow.., columns tcol.. of that 128-byte-swizzled 64 x 64 tile; keep_fp32 =
// false leaves the fp32 copy out.
template <int LDA, int K, int NNT = 2>
__device__ __forceinline__ void warp_gemm16(const float *Am, const float *Bm, float *Cm, float sign, int lane,
                                            uint8_t *tt = nullptr, int trow = 0, int tcol = 0,
                                            bool keep_fp32 = true) {
    const int g = lane >> 2, q = lane & 3;
    float acc[NNT][4] = {};
#pragma unroll
    for (int k0 = 0; k0 < K; k0 += 8) {
        const uint32_t a[4] = {to_tf32(Am[g * LDA + k0 + q]), to_tf32(Am[(g + 8) * LDA + k0 + q]),
                               to_tf32(Am[g * LDA + k0 + q + 4]), to_tf32(Am[(g + 8) * LDA + k0 + q + 4])};
#pragma unroll
        for (int nt = 0; nt < NNT; ++nt) {
            const uint32_t bf[2] = {to_tf32(Bm[(k0 + q) * LDA + 8 * nt + g]), to_tf32(Bm[(k0 + q + 4) * LDA + 8 * nt + g])};
            mma_tf32(acc[nt], a, bf);
        }
    }
#pragma unroll
    for (int nt = 0; nt < NNT; ++nt) {
        if (keep_fp32) {
            *reinterpret_cast<float2 *>(Cm + g * LDA + 8 * nt + 2 * q) = make_float2(sign * acc[nt][0], sign * acc[nt][1]);
            *reinterpret_cast<float2 *>(Cm + (g + 8) * LDA + 8 * nt + 2 * q) =
                make_float2(sign * acc[nt][2], sign * acc[nt][3]);
        }
        if (tt != nullptr) {
            const uint32_t c = static_cast<uint32_t>(tcol + 8 * nt + 2 * q);
            *reinterpret_cast<uint32_t *>(tt + sw128_off(trow + g, c)) = pack_bf16x2(sign * acc[nt][0], sign * acc[nt][1]);
            *reinterpret_cast<uint32_t *>(tt + sw128_off(trow + g + 8, c)) = pack_bf16x2(sign * acc[nt][2], sign * acc[nt][3]);
        }
    }
}

// T = (I + A)^{-1} for a strictly lower 64x64 A held in fp32 in sA (row
// stride LDA), in place, by 128 threads (4 warps):
//   1. each 16x16 diagonal block D_k = (I + A_kk)^{-1} by right-looking
//      forward substitution in fp32, warp k for block k, two lanes a column;
//   2. 16 -> 32: T_{2p+1,2p} = -D_{2p+1} (A_{2p+1,2p} D_{2p}), p = 0, 1
//      (warp p);
//   3. 32 -> 64: T_ba = -T_b (A_ba T_a) with a = rows/cols 0-31, b = 32-63
//      (warp w: rows 16 (w % 2), columns 16 (w / 2) of each product).
// The block products run on the tensor cores (mma.sync, tf32 inputs, fp32
// accumulation); T is rounded to bf16, which dominates the tf32 input
// rounding.  The intermediate products go to the upper-right 32x32 block of
// the scratch.  T also goes, as bf16, to the 128-byte-swizzled MMA tile `tt`
// as each block becomes final: the diagonal blocks during step 2, T_{2p+1,2p}
// and T_ba from the products' fragments.  Blocks above the diagonal of `tt`
// are never written here: they keep the zeros the kernel's setup wrote.
// `bar` is a named barrier over exactly these 128 threads; they fence their
// tile writes for the tensor core before returning.
template <int LDA>
__device__ __forceinline__ void unit_lower_inverse64(float *sA, uint8_t *tt, int t, int bar) {
    const int w = t >> 5, lane = t & 31;
    {   // 1. diagonal blocks: warp b takes block b; lanes 2j and 2j + 1 share column j
        // (rows of parity lane % 2), right-looking: row i of the column is final
        // once the rows above have applied their terms, and is broadcast
        const int R = 16 * w, j = lane >> 1, hh = lane & 1;
        const float *blk = sA + R * LDA + R;
        float acc[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) acc[m] = (2 * m + hh == j) ? 1.f : 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float xi = __shfl_sync(0xffffffffu, acc[i >> 1], (lane & ~1) | (i & 1));
#pragma unroll
            for (int m = i >> 1; m < 8; ++m) {
                const int r = 2 * m + hh;
                if (r > i) acc[m] = fmaf(-blk[r * LDA + i], xi, acc[m]);
            }
        }
        named_bar(bar, 128);   // every column has read A's block before D overwrites it
#pragma unroll
        for (int m = 0; m < 8; ++m) sA[(R + 2 * m + hh) * LDA + R + j] = acc[m];
        named_bar(bar, 128);
    }
    {   // 2. 16 -> 32: pair p = w % 2 (Y_p in rows 16p.., cols 32..), 8-column half w / 2
        const int pr = w & 1, half = 8 * (w >> 1), R = 32 * pr;
        float *Y = sA + (16 * pr) * LDA + 32;
        warp_gemm16<LDA, 16, 1>(sA + (R + 16) * LDA + R, sA + R * LDA + R + half, Y + half, 1.f, lane);
        named_bar(bar, 128);   // both halves of each Y_p are written
        warp_gemm16<LDA, 16, 1>(sA + (R + 16) * LDA + R + 16, Y + half, sA + (R + 16) * LDA + R + half, -1.f, lane,
                                tt, R + 16, R + half);
        // the diagonal blocks to the tile, 8 columns a thread
        {
            const int c = t;   // the 128 8-column pieces of the four blocks
            const int b = c >> 5, row = 16 * b + ((c >> 1) & 15), col0 = 16 * b + 8 * (c & 1);
            const float4 a = *reinterpret_cast<const float4 *>(sA + row * LDA + col0);
            const float4 d = *reinterpret_cast<const float4 *>(sA + row * LDA + col0 + 4);
            *reinterpret_cast<uint4 *>(tt + sw128_chunk(row, col0 >> 3)) =
                make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(d.x, d.y), pack_bf16x2(d.z, d.w));
        }
    }
    named_bar(bar, 128);
    {   // 3. 32 -> 64: Y = A_ba T_a into rows 0-31, cols 32-63; then T_ba = -T_b Y (to the tile only)
        const int rm = 16 * (w & 1), cn = 16 * (w >> 1);
        warp_gemm16<LDA, 32>(sA + (32 + rm) * LDA, sA + cn, sA + rm * LDA + 32 + cn, 1.f, lane);
        named_bar(bar, 128);
        warp_gemm16<LDA, 32>(sA + (32 + rm) * LDA + 32, sA + 32 + cn, nullptr, -1.f, lane, tt, 32 + rm, cn, false);
        named_bar(bar, 128);
    }
    fence_proxy_async_smem();   // MMA3 and MMA_T read the tile
}

// 8 bf16 products of two 16-byte vectors, rounded back to bf16 (packed bf16x2
// multiplies: the exact product rounded once, as fp32 multiply + rounding).
__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
__device__ __forceinline__ uint4 mul_bf16x8(const uint4 &a, const uint4 &b) {
    return make_uint4(mul_bf16x2(a.x, b.x), mul_bf16x2(a.y, b.y), mul_bf16x2(a.z, b.z), mul_bf16x2(a.w, b.w));
}
// 2^x (MUFU approximation, flush-to-zero).
__device__ __forceinline__ float ex2(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// log_alpha of one chunk for the prep thread g (channel quad p = g % (DK/4),
// rows R hb .. R hb + R - 1 with hb = g / (DK/4)), straight from HBM into
// registers; rows past the sequence end read as zero (no decay on padding).
template <int DK>
struct PrepLA {
    static constexpr int NP = DK / 4, NB = 128 / NP, R = 64 / NB;
    uint2 v[R];
    // chunk n of the sequence made of tokens [tok0, tok0 + len); key head h of H
    __device__ __forceinline__ void load(const __nv_bfloat16 *la, long tok0, int n, int h, int len, int H, int g) {
        const int p = g % NP, hb = g / NP;
#pragma unroll
        for (int i = 0; i < R; ++i) {
            const int r = n * 64 + hb * R + i;
            const uint2 *src = reinterpret_cast<const uint2 *>(la + ((tok0 + r) * H + h) * DK + 4 * p);
            v[i] = (r < len && GDN2_IN_BOUNDS(kBufLA, src, 8)) ? __ldg(src) : make_uint2(0u, 0u);
        }
    }
};

// Prep of one chunk by 128 threads (thread g): the per-channel cumulative
// log-decay G (fp32, in row order, kept as G log2(e)), the reference point
// ref = (G_0 + G_C) / 2 and, in place in the TMA tiles,
//     Q~ = q.exp(G - ref),  E = b.k.exp(G - ref),  K~ = k.exp(ref - G),
// plus exp(G_C - ref) and exp(ref) into gc[0..127] and gc[128..255].  A chunk whose
// span G_0 - G_C passes kMaxChunkSpan2 in any channel sets *stop_at = chunk (its
// tiles are then never used).  Thread g owns the channel quad
// p = g % (DK/4) over a block of R consecutive rows (its log_alpha values in
// `law`); the running sum enters a block with the totals of the blocks above
// it (exchanged through `carry` and named barrier `bar` over the 128
// threads).  A half-warp covers 16 consecutive quads = one 128-byte swizzled
// row, so the 8-byte shared accesses are conflict-free.
// PACKED takes the products as packed bf16x2 multiplies of the bf16 inputs by
// the bf16-rounded factors (about one more bf16 rounding per operand).
// With PREP, q, k, b arrive raw: each row of q and k is scaled by
// 1 / sqrt(sum^2 + l2_eps) (a pre-pass: thread t sums row t % 64 of q (t < 64)
// or of k, and leaves the factor in `nrm`) and b becomes sigmoid(b) (x2 with
// neg_eigval).
// Rows at or past `rows_valid` (the end of a packed sequence inside the
// chunk) hold the next sequence's tokens: they are cleared in the raw q, b, k
// tiles first, which makes them the same exact no-ops as padding.  This runs
// only on a sequence's partial last chunk and leaves the loop below as is.
template <int DK, bool PREP = false, bool VARLEN = false, bool PACKED = false>
__device__ __forceinline__ void prep_chunk(uint8_t *smem, uint32_t oqe, uint32_t okt, const PrepLA<DK> &law,
                                           float *gc, float *carry, int g, int bar, int chunk,
                                           volatile int *stop_at, const FuseArgs &fz = {},
                                           float2 *nrm = nullptr, int rows_valid = 64) {
    constexpr int NP = PrepLA<DK>::NP, NB = PrepLA<DK>::NB, R = PrepLA<DK>::R;
    static_assert(NB * R == 64 && NB <= 8, "prep split");
    const int p = g % NP, hb = g / NP;
    const int kb = p >> 4, cb = (p & 15) * 8;   // channel block, byte in the 128-byte row
    uint8_t *q_t = smem + oqe + kb * 16384, *e_t = q_t + 8192, *k_t = smem + okt + kb * 8192;
    auto off = [&](int r) { return r * 128 + ((((cb >> 4) ^ r) & 7) << 4) + (cb & 15); };
    if (VARLEN && rows_valid < 64) {   // uniform over the 128 threads
        // a swizzled row keeps its own 128 bytes: clear bytes [128 rows_valid, 8192)
        // of each 8 KB q, b and k sub-tile
        const int n16 = (64 - rows_valid) * 8;
        for (int idx = g; idx < 3 * (DK / 64) * n16; idx += 128) {
            const int tile = idx / n16, piece = idx - tile * n16, kb2 = tile / 3, which = tile - kb2 * 3;
            uint8_t *base = (which == 2) ? smem + okt + kb2 * 8192 : smem + oqe + kb2 * 16384 + which * 8192;
            *reinterpret_cast<uint4 *>(base + rows_valid * 128 + piece * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
        named_bar(bar, 128);
    }
    if constexpr (PREP) {   // 1 / |row| of q (threads 0-63) and k (64-127)
        const int r = g & 63;
        const uint8_t *base = (g < 64) ? smem + oqe : smem + okt;
        const uint32_t kstride = (g < 64) ? 16384u : 8192u;
        float ss[4] = {0.f, 0.f, 0.f, 0.f};   // four partial sums: short dependency chains
#pragma unroll
        for (int c8 = 0; c8 < DK / 8; ++c8) {
            uint32_t a0, a1, a2, a3;
            ld_shared_v4(smem_u32(base + (c8 >> 3) * kstride) + sw128_chunk(r, c8 & 7), a0, a1, a2, a3);
            const uint32_t aa[4] = {a0, a1, a2, a3};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                ss[e] = fmaf(bf16_lo(aa[e]), bf16_lo(aa[e]), ss[e]);
                ss[e] = fmaf(bf16_hi(aa[e]), bf16_hi(aa[e]), ss[e]);
            }
        }
        reinterpret_cast<float *>(nrm)[2 * r + (g >> 6)] = l2_inv((ss[0] + ss[1]) + (ss[2] + ss[3]), fz.l2_eps);
    }
    // running sums in log2 units (G log2(e)), so that exp(+-G) = 2^(+-sum)
    constexpr float kLog2e = 1.4426950408889634f;
    float sum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < R; ++i) {
        sum[0] = fmaf(bf16_lo(law.v[i].x), kLog2e, sum[0]);
        sum[1] = fmaf(bf16_hi(law.v[i].x), kLog2e, sum[1]);
        sum[2] = fmaf(bf16_lo(law.v[i].y), kLog2e, sum[2]);
        sum[3] = fmaf(bf16_hi(law.v[i].y), kLog2e, sum[3]);
    }
    float4 *carry4 = reinterpret_cast<float4 *>(carry);
    carry4[hb * NP + p] = make_float4(sum[0], sum[1], sum[2], sum[3]);
    if (hb == 0)   // row 0 on its own: the reference point is taken from G_0 and G_C
        carry4[NB * NP + p] = make_float4(bf16_lo(law.v[0].x) * kLog2e, bf16_hi(law.v[0].x) * kLog2e,
                                          bf16_lo(law.v[0].y) * kLog2e, bf16_hi(law.v[0].y) * kLog2e);
    named_bar(bar, 128);
    // Reference point ref = (G_0 + G_C) / 2 per channel: the operands are scaled by
    // 2^(G_r - ref) and 2^(ref - G_r), both within 2^(+-span / 2) with span = G_0 - G_C
    // (the decay of rows 1..63; row 0's own decay only scales the incoming state).
    // The running sum enters this thread's rows at (sum of the blocks above) - ref
    //   = sum_h2 (h2 < hb ? 1/2 : -1/2) carry[h2] - G_0 / 2.
    {
        const float4 r4 = carry4[NB * NP + p];
        sum[0] = -0.5f * r4.x;
        sum[1] = -0.5f * r4.y;
        sum[2] = -0.5f * r4.z;
        sum[3] = -0.5f * r4.w;
    }
#pragma unroll
    for (int h2 = 0; h2 < NB; ++h2) {
        const float4 c4 = carry4[h2 * NP + p];
        const float wgt = h2 < hb ? 0.5f : -0.5f;
        sum[0] = fmaf(wgt, c4.x, sum[0]);
        sum[1] = fmaf(wgt, c4.y, sum[1]);
        sum[2] = fmaf(wgt, c4.z, sum[2]);
        sum[3] = fmaf(wgt, c4.w, sum[3]);
    }
    // rows in batches of RB, software-pipelined: the tiles are rewritten in
    // place, so the compiler keeps every load behind the earlier stores; the
    // next batch's loads are therefore issued here before this batch is stored
    // (they read other rows)
    constexpr int RB = 2;
    uint2 qw[RB], kw[RB], bw[RB];
#pragma unroll
    for (int j = 0; j < RB; ++j) {
        const int oj = off(hb * R + j);
        qw[j] = *reinterpret_cast<const uint2 *>(q_t + oj);
        kw[j] = *reinterpret_cast<const uint2 *>(k_t + oj);
        bw[j] = *reinterpret_cast<const uint2 *>(e_t + oj);
    }
#pragma unroll
    for (int i0 = 0; i0 < R; i0 += RB) {
        uint2 qn[RB], kn[RB], bn[RB];
        if (i0 + RB < R) {
#pragma unroll
            for (int j = 0; j < RB; ++j) {
                const int oj = off(hb * R + i0 + RB + j);
                qn[j] = *reinterpret_cast<const uint2 *>(q_t + oj);
                kn[j] = *reinterpret_cast<const uint2 *>(k_t + oj);
                bn[j] = *reinterpret_cast<const uint2 *>(e_t + oj);
            }
        }
        int o[RB];
#pragma unroll
        for (int j = 0; j < RB; ++j) o[j] = off(hb * R + i0 + j);
#pragma unroll
        for (int j = 0; j < RB; ++j) {
            float rq = 1.f, rk = 1.f, bs = 1.f;
            if constexpr (PREP) {
                const float2 nr = nrm[hb * R + i0 + j];
                rq = nr.x;
                rk = nr.y;
                bs = fz.neg_eigval ? 2.f : 1.f;
            }
            const uint2 la2 = law.v[i0 + j];
            sum[0] = fmaf(bf16_lo(la2.x), kLog2e, sum[0]);
            sum[1] = fmaf(bf16_hi(la2.x), kLog2e, sum[1]);
            sum[2] = fmaf(bf16_lo(la2.y), kLog2e, sum[2]);
            sum[3] = fmaf(bf16_hi(la2.y), kLog2e, sum[3]);
            const uint32_t qv[2] = {qw[j].x, qw[j].y}, kv[2] = {kw[j].x, kw[j].y}, bv[2] = {bw[j].x, bw[j].y};
            uint32_t oq[2], oe[2], ok[2];
            if constexpr (PACKED) {
                // the scale factors rounded to bf16 and the products taken as packed
                // bf16x2 multiplies (each rounded once): fewer instructions, about one
                // more bf16 rounding per operand
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t gap = pack_bf16x2(ex2(sum[2 * h]), ex2(sum[2 * h + 1]));
                    const uint32_t ivp = pack_bf16x2(ex2(-sum[2 * h]), ex2(-sum[2 * h + 1]));
                    oq[h] = mul_bf16x2(qv[h], gap);
                    oe[h] = mul_bf16x2(mul_bf16x2(bv[h], kv[h]), gap);
                    ok[h] = mul_bf16x2(kv[h], ivp);
                }
            } else {
                // fp32 products, two channels per paired instruction (same roundings)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float2 ga = make_float2(ex2(sum[2 * h]), ex2(sum[2 * h + 1]));
                    const float2 iv = make_float2(ex2(-sum[2 * h]), ex2(-sum[2 * h + 1]));
                    float2 k2 = make_float2(bf16_lo(kv[h]), bf16_hi(kv[h]));
                    float2 b2 = make_float2(bf16_lo(bv[h]), bf16_hi(bv[h]));
                    float2 q2 = make_float2(bf16_lo(qv[h]), bf16_hi(qv[h]));
                    if constexpr (PREP) {
                        k2 = mul_f32x2(k2, make_float2(rk, rk));
                        q2 = mul_f32x2(q2, make_float2(rq, rq));
                        // sigmoid(x) = 0.5 + 0.5 tanh(x / 2), times bs
                        const float2 hx = mul_f32x2(b2, make_float2(0.5f, 0.5f));
                        float2 th;
                        asm("tanh.approx.f32 %0, %1;" : "=f"(th.x) : "f"(hx.x));
                        asm("tanh.approx.f32 %0, %1;" : "=f"(th.y) : "f"(hx.y));
                        const float hb = 0.5f * bs;
                        b2 = fma_f32x2(th, make_float2(hb, hb), make_float2(hb, hb));
                    }
                    const float2 xq = mul_f32x2(q2, ga), xe = mul_f32x2(mul_f32x2(b2, k2), ga), xk = mul_f32x2(k2, iv);
                    oq[h] = pack_bf16x2(xq.x, xq.y);
                    oe[h] = pack_bf16x2(xe.x, xe.y);
                    ok[h] = pack_bf16x2(xk.x, xk.y);
                }
            }
            *reinterpret_cast<uint2 *>(q_t + o[j]) = make_uint2(oq[0], oq[1]);
            *reinterpret_cast<uint2 *>(e_t + o[j]) = make_uint2(oe[0], oe[1]);
            *reinterpret_cast<uint2 *>(k_t + o[j]) = make_uint2(ok[0], ok[1]);
        }
        if (i0 + RB < R) {
#pragma unroll
            for (int j = 0; j < RB; ++j) {
                qw[j] = qn[j];
                kw[j] = kn[j];
                bw[j] = bn[j];
            }
        }
    }
    if (hb == NB - 1) {
        // the last rows end at G_C - ref = -span / 2: 2^(G_C - ref) is the factor applied
        // after the state update, 2^ref = 2^(G_0 - span / 2) the scale of the incoming state
        const float4 r4 = carry4[NB * NP + p];
        const float g0[4] = {r4.x, r4.y, r4.z, r4.w};
        bool out = false;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            out |= !(-2.f * sum[e] <= kMaxChunkSpan2);   // also catches NaN from infinite decays
            gc[4 * p + e] = ex2(sum[e]);
            gc[128 + 4 * p + e] = ex2(g0[e] + sum[e]);
        }
        if (out) *stop_at = chunk;   // every writer stores the same value
    }
    fence_proxy_async_smem();
}

// ------------------------------------------------ second erase direction (QED)
// With the query-derived erase direction ("The Query Knows What to Forget",
// mlsanity 2608.13668, abstract; reading in qed.cuh) a chunk is 32 tokens and
// 64 pseudo-rows: row 2t is token t's key (erase b_t.k_t, value w_t.v_t), row
// 2t + 1 its query direction u_t (erase c_t.u_t, value 0).  Both rows of a token
// read the state before the token, so A is strictly lower by token, and only
// the 32 token rows carry a query (P and O rows 0-31; rows 32-63 unused).  The
// tiles keep their 64-row shapes; the TMA brings the 32 token rows in as
//     Q~ rows 0-31: q      Q~ rows 32-63: c      E rows 32-63: b
//     K~ rows 32-63: k     v rows 32-63: v       w rows 0-31: w
// and the prep and W.V expand them in place into the pseudo-rows.

// log_alpha of one 32-token chunk for prep thread c (key channel c): 32 bf16
// values, one per register and untouched until the prep uses them (a whole
// iteration later), so the loads' latency stays hidden; tokens past the
// sequence end read as 0.
template <int DK>
struct PrepLAQ {
    uint32_t v[32];
    __device__ __forceinline__ void load(const __nv_bfloat16 *la, long tok0, int n, int h, int len, int H, int c) {
        const unsigned short *p = reinterpret_cast<const unsigned short *>(la);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int r = n * 32 + i;
            const unsigned short *src = p + ((tok0 + r) * H + h) * DK + c;
            v[i] = (c < DK && r < len && GDN2_IN_BOUNDS(kBufLA, src, 2)) ? static_cast<uint32_t>(__ldg(src)) : 0u;
        }
    }
    __device__ __forceinline__ float get(int i) const { return __uint_as_float(v[i] << 16); }
};

__device__ __forceinline__ void st_shared_u16(uint32_t addr, unsigned short x) {
    asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(x) : "memory");
}
__device__ __forceinline__ unsigned short bf16_bits(float x) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// Prep of one QED chunk by 128 threads (thread g):
//  1. per token t (warp g / 32 takes tokens 8 (g / 32) .., lane = channel quad):
//     coef_t = q.k / k.k (0 when k = 0), r = q - coef_t k, nu_t = 1 / sqrt(r.r + eps)
//     (0 when that is 0), into scal[t];
//  2. thread g = key channel c: the running log2-decay G_t over the 32 tokens,
//     ref = (G_0 + G_31) / 2, and, in place, u_t = (q_t - coef_t k_t) nu_t and
//     Q~_t = q.2^(G-ref), E_2t = b.k.2^(G-ref), E_2t+1 = c.u.2^(G-ref),
//     K~_2t = k.2^(ref-G), K~_2t+1 = u.2^(ref-G).
// Q~ rows 32-63 keep the raw c: the P read-out masks those rows to zero and the
// rows of X they reach (32-63) are never stored, so they need no clearing.
// Every read and write of channel c in step 2 is thread c's, in token order, so
// the pseudo-row writes of token t only ever overwrite raw rows of tokens
// <= t that the thread has already read.  gc and the stop flag as prep_chunk.
template <int DK>
__device__ __forceinline__ void prep_chunk_qed(uint8_t *smem, uint32_t oqe, uint32_t okt, const PrepLAQ<DK> &law,
                                               float *gc, float2 *scal, int g, int bar, int chunk,
                                               volatile int *stop_at, float qed_eps) {
    {   // 1. per-token coefficients of the query direction
        const int w = g >> 5, l = g & 31, p = l;   // channel quad p (4 channels) of tokens 8 w ..
        const bool act = 4 * p < DK;
        const int kb = (4 * p) >> 6, cb = ((4 * p) & 63) * 2;   // channel block, byte in the 128-byte row
        const uint8_t *qt = smem + oqe + kb * 16384, *kt = smem + okt + kb * 8192;
        auto off = [&](int r) { return r * 128 + ((((cb >> 4) ^ r) & 7) << 4) + (cb & 15); };
        // four tokens at a time, their reductions interleaved (independent shuffle chains)
#pragma unroll 1
        for (int i0 = 0; i0 < 8; i0 += 4) {
            uint2 q2[4], k2[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int t = 8 * w + i0 + j;
                q2[j] = act ? *reinterpret_cast<const uint2 *>(qt + off(t)) : make_uint2(0u, 0u);
                k2[j] = act ? *reinterpret_cast<const uint2 *>(kt + off(32 + t)) : make_uint2(0u, 0u);
            }
            float qk[4], kk[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float qv[4] = {bf16_lo(q2[j].x), bf16_hi(q2[j].x), bf16_lo(q2[j].y), bf16_hi(q2[j].y)};
                const float kv[4] = {bf16_lo(k2[j].x), bf16_hi(k2[j].x), bf16_lo(k2[j].y), bf16_hi(k2[j].y)};
                qk[j] = 0.f;
                kk[j] = 0.f;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    qk[j] = fmaf(qv[e], kv[e], qk[j]);
                    kk[j] = fmaf(kv[e], kv[e], kk[j]);
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    qk[j] += __shfl_xor_sync(0xffffffffu, qk[j], o);
                    kk[j] += __shfl_xor_sync(0xffffffffu, kk[j], o);
                }
            float coef[4], rr[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                coef[j] = kk[j] > 0.f ? qk[j] / kk[j] : 0.f;
                const float qv[4] = {bf16_lo(q2[j].x), bf16_hi(q2[j].x), bf16_lo(q2[j].y), bf16_hi(q2[j].y)};
                const float kv[4] = {bf16_lo(k2[j].x), bf16_hi(k2[j].x), bf16_lo(k2[j].y), bf16_hi(k2[j].y)};
                rr[j] = 0.f;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float r = qv[e] - coef[j] * kv[e];
                    rr[j] = fmaf(r, r, rr[j]);
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
#pragma unroll
                for (int j = 0; j < 4; ++j) rr[j] += __shfl_xor_sync(0xffffffffu, rr[j], o);
            if (l < 4) {   // lane j writes token 8 w + i0 + j (selects keep the arrays in registers)
                const float cf = l == 0 ? coef[0] : l == 1 ? coef[1] : l == 2 ? coef[2] : coef[3];
                const float den = (l == 0 ? rr[0] : l == 1 ? rr[1] : l == 2 ? rr[2] : rr[3]) + qed_eps;
                scal[8 * w + i0 + l] = make_float2(cf, den > 0.f ? rsqrtf(den) : 0.f);
            }
        }
    }
    named_bar(bar, 128);
    constexpr float kLog2e = 1.4426950408889634f;
    const int c = g;
    if (c < DK) {
        float total = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) total = fmaf(law.get(i), kLog2e, total);
        const float g0 = law.get(0) * kLog2e;
        float sum = -0.5f * (g0 + total);   // the running sum enters at -ref
        const int kb = c >> 6, cc = c & 63;
        const uint32_t qt = smem_u32(smem + oqe + kb * 16384), et = qt + 8192u, kt = smem_u32(smem + okt + kb * 8192);
        // the column part of the swizzled offset for each row phase (row & 7, a
        // constant in the unrolled loop): element (row, cc) sits at row * 128 + cx[row & 7]
        uint32_t cx[8];
#pragma unroll
        for (int r8 = 0; r8 < 8; ++r8) cx[r8] = ((((cc >> 3) ^ r8) & 7) << 4) + ((cc & 7) << 1);
        auto at = [&](int row) { return static_cast<uint32_t>(row * 128) + cx[row & 7]; };
#pragma unroll
        for (int t = 0; t < 32; ++t) {
            sum = fmaf(law.get(t), kLog2e, sum);
            const float ga = ex2(sum), iv = ex2(-sum);
            const float q = ld_shared_bf16(qt + at(t));
            const float cg = ld_shared_bf16(qt + at(32 + t));
            const float k = ld_shared_bf16(kt + at(32 + t));
            const float b = ld_shared_bf16(et + at(32 + t));
            const float2 sc = scal[t];
            const float u = (q - sc.x * k) * sc.y;
            st_shared_u16(qt + at(t), bf16_bits(q * ga));   // rows 32-63 keep c (see below)
            st_shared_u16(et + at(2 * t), bf16_bits(b * k * ga));
            st_shared_u16(et + at(2 * t + 1), bf16_bits(cg * u * ga));
            st_shared_u16(kt + at(2 * t), bf16_bits(k * iv));
            st_shared_u16(kt + at(2 * t + 1), bf16_bits(u * iv));
        }
        // sum ends at G_31 - ref = -span / 2 (span: the decay of tokens 1..31)
        gc[c] = ex2(sum);
        gc[128 + c] = ex2(g0 + sum);
        if (!(-2.f * sum <= kMaxChunkSpan2)) *stop_at = chunk;
    }
    fence_proxy_async_smem();
}

// Packed sequences: grid slot z runs the sequence of length rank z (longest
// first, ties by index), so that blocks, which start in z order, begin with
// the long sequences and the short ones fill in behind them (longest-
// processing-time-first scheduling).  Every CTA ranks the lengths itself in
// `scratch` (shared memory that the setup clears afterwards): warp w takes
// candidates i = w, w + warps, ..., its lanes count the sequences ahead of i.
// Up to kMaxRankedSeqs sequences; beyond that slot z runs sequence z.
constexpr int kMaxRankedSeqs = 1024;
__device__ __forceinline__ int longest_first_sequence(const int *__restrict__ cu, int nseq, int slot, int *scratch) {
    if (nseq <= 1 || nseq > kMaxRankedSeqs) return slot;
    int *lens = scratch, *pick = scratch + kMaxRankedSeqs;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    for (int i = tid; i < nseq; i += blockDim.x)
        lens[i] = (GDN2_IN_BOUNDS(kBufCU, cu + i, 8)) ? cu[i + 1] - cu[i] : 0;
    if (tid == 0) *pick = slot;   // a total order always has one sequence of rank `slot`
    __syncthreads();
    for (int i = warp; i < nseq; i += nwarps) {
        const int li = lens[i];
        int ahead = 0;
        for (int j = lane; j < nseq; j += 32) {
            const int lj = lens[j];
            ahead += (lj > li || (lj == li && j < i)) ? 1 : 0;
        }
        ahead = __reduce_add_sync(0xffffffffu, ahead);
        if (lane == 0 && ahead == slot) *pick = i;
    }
    __syncthreads();
    const int r = *pick;
    __syncthreads();   // everyone has read it before the scratch is reused
    return r;
}

// N consecutive bf16 values (N = 2 or 4) read with one 4- or 8-byte load.
template <int N>
struct BfVec {
    static_assert(N == 2 || N == 4, "bf16 vector");
    uint32_t w[N / 2];
    __device__ __forceinline__ void load(const __nv_bfloat16 *p, int buf) {
        if (!GDN2_IN_BOUNDS(buf, p, 2 * N)) {
#pragma unroll
            for (int e = 0; e < N / 2; ++e) w[e] = 0u;
            return;
        }
        if constexpr (N == 4) {
            const uint2 x = __ldg(reinterpret_cast<const uint2 *>(p));
            w[0] = x.x;
            w[1] = x.y;
        } else {
            w[0] = __ldg(reinterpret_cast<const unsigned int *>(p));
        }
    }
    __device__ __forceinline__ float get(int e) const { return (e & 1) ? bf16_hi(w[e >> 1]) : bf16_lo(w[e >> 1]); }
};

// Raw token pointers for the token tail (the main loop reads through TMA maps).
struct TailArgs {
    const __nv_bfloat16 *q, *k, *b, *v, *w;
    const __nv_bfloat16 *c = nullptr;   // QED: the second erase gate
    float qed_eps = 0.f;                 // QED: epsilon of the direction's norm
};

// Token tail: a chunk whose decay span passes kMaxChunkSpan2, and every later
// chunk of its sequence, run here token by token, straight from the step
//     r_j = sum_c (b_c k_c alpha_c) S_cj,   p_j = sum_c (q_c alpha_c) S_cj,
//     u_j = w_j v_j - r_j,   S_cj <- alpha_c S_cj + k_c u_j,   o_j = p_j + (q . k) u_j
// with alpha = exp(log_alpha) per token, so a decay of any strength is exact to
// fp32 rounding.  `smem` holds the state at the start of token t_begin as fp32
// [DK][NV + 4] (row c, column j).
//   warps 0-7   arithmetic: lane = 8 cb + rb; thread (warp, cb, rb) holds rows
//               rb, rb + 8, ... (DK / 8 of them) of the NV / 32 columns
//               (4 warp + cb) NV / 32 .. in registers; the column sums over the
//               rows reduce across the 8 rb lanes by shuffles
//   warps 8-12  stage the inputs of TB tokens at a time into one of two
//               buffers (warp 8 + s: tokens s, s + 5, ...), handed over with
//               named barriers (full: staging arrives, arithmetic waits; empty:
//               the other way round)
// Every thread of the block calls it.
template <int DK, int NV, bool PREP, bool EPI>
__device__ __noinline__ void tc_token_tail(uint8_t *smem, const TailArgs ta, const __nv_bfloat16 *__restrict__ la,
                                           __nv_bfloat16 *__restrict__ o, float *__restrict__ S_T, long tok0,
                                           int t_begin, int len, int h, int H, int hv, int HV, int j0, int d_v,
                                           long head, const FuseArgs fz) {
    constexpr int TB = 16, LS = NV + 4;
    constexpr int RR = DK / 8, CJ = NV / 32;      // rows and columns of S per arithmetic thread
    constexpr int CPL = DK / 32, JPL = NV / 32;   // channels / columns per lane when staging
    constexpr int kStage = 5, kAll = kTcThreads;  // staging warps; threads on the hand-off barriers
    constexpr int BAR_FULL = 5, BAR_EMPTY = 7, BAR_MATH = 9;   // ids 5-6, 7-8 by buffer; 9: arithmetic only
    const float *sS = reinterpret_cast<const float *>(smem);
    float4 *rowd = reinterpret_cast<float4 *>(smem + DK * LS * 4);    // [2][TB][DK]: alpha, b k alpha, q alpha, k
    float2 *cold = reinterpret_cast<float2 *>(rowd + 2 * TB * DK);     // [2][TB][NV]: w v, gate
    float *qkb = reinterpret_cast<float *>(cold + 2 * TB * NV);        // [2][TB]: q . k
    float *obuf = qkb + 2 * TB;                                        // [TB][NV] (EPI)
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nb = (len - t_begin + TB - 1) / TB;   // batches
    if (warp < 8) {
        // ============================================================ arithmetic
        const int rb = lane & 7, cb = lane >> 3, jb = (4 * warp + cb) * CJ;
        float Sr[RR][CJ];
#pragma unroll
        for (int i = 0; i < RR; ++i)
#pragma unroll
            for (int x = 0; x < CJ; ++x) Sr[i][x] = sS[(8 * i + rb) * LS + jb + x];
        for (int k = 0; k < nb; ++k) {
            const int buf = k & 1, tb = t_begin + k * TB, nt = min(TB, len - tb);
            named_bar(BAR_FULL + buf, kAll);
            const float4 *rdb = rowd + buf * TB * DK;
            for (int tt = 0; tt < nt; ++tt) {
                const float4 *rd = rdb + tt * DK;
                float r[CJ], pq[CJ];
#pragma unroll
                for (int x = 0; x < CJ; ++x) r[x] = pq[x] = 0.f;
#pragma unroll
                for (int i = 0; i < RR; ++i) {
                    const float4 xr = rd[8 * i + rb];
#pragma unroll
                    for (int x = 0; x < CJ; ++x) {
                        r[x] = fmaf(xr.y, Sr[i][x], r[x]);
                        pq[x] = fmaf(xr.z, Sr[i][x], pq[x]);
                    }
                }
#pragma unroll
                for (int off = 1; off < 8; off <<= 1)
#pragma unroll
                    for (int x = 0; x < CJ; ++x) {
                        r[x] += __shfl_xor_sync(0xffffffffu, r[x], off);
                        pq[x] += __shfl_xor_sync(0xffffffffu, pq[x], off);
                    }
                const float qk = qkb[buf * TB + tt];
                float u[CJ], ov[CJ];
#pragma unroll
                for (int x = 0; x < CJ; ++x) {
                    u[x] = cold[(buf * TB + tt) * NV + jb + x].x - r[x];
                    ov[x] = fmaf(qk, u[x], pq[x]);
                }
#pragma unroll
                for (int i = 0; i < RR; ++i) {
                    const float4 xr = rd[8 * i + rb];
#pragma unroll
                    for (int x = 0; x < CJ; ++x) Sr[i][x] = fmaf(xr.x, Sr[i][x], xr.w * u[x]);
                }
                if (rb == 0) {
                    if constexpr (EPI) {
#pragma unroll
                        for (int x = 0; x < CJ; ++x) obuf[tt * NV + jb + x] = ov[x];
                    } else {
                        __nv_bfloat16 *dst = o + ((tok0 + tb + tt) * HV + hv) * (long)d_v + j0 + jb;
                        if (GDN2_IN_BOUNDS(kBufO, dst, 2 * CJ)) {
#pragma unroll
                            for (int x = 0; x < CJ; x += 2)
                                *reinterpret_cast<uint32_t *>(dst + x) = pack_bf16x2(ov[x], ov[x + 1]);
                        }
                    }
                }
            }
            if constexpr (EPI) {   // y = o / sqrt(mean(o^2) + eps) . weight . silu(gate), a warp per token
                named_bar(BAR_MATH, 256);
                for (int tt = warp; tt < nt; tt += 8) {
                    float ss = 0.f;
#pragma unroll
                    for (int e = 0; e < JPL; ++e) {
                        const float x = obuf[tt * NV + lane + 32 * e];
                        ss = fmaf(x, x, ss);
                    }
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
                    const float inv = rsqrtf(ss / (float)NV + fz.norm_eps);
                    const long vro = ((tok0 + tb + tt) * HV + hv) * (long)d_v + j0;
#pragma unroll
                    for (int e = 0; e < JPL; ++e) {
                        const int jj = lane + 32 * e;
                        const float gt = cold[(buf * TB + tt) * NV + jj].y;
                        if (!GDN2_IN_BOUNDS(kBufO, o + vro + jj, 2) || !GDN2_IN_BOUNDS(kBufNW, fz.norm_weight + j0 + jj, 4))
                            continue;
                        o[vro + jj] = __float2bfloat16_rn(obuf[tt * NV + jj] * inv * fz.norm_weight[j0 + jj] * gt *
                                                          sigmoid_f32(gt));
                    }
                }
                named_bar(BAR_MATH, 256);   // obuf is rewritten by the next batch
            }
            if (k + 2 < nb) named_bar_arrive(BAR_EMPTY + buf, kAll);   // the staging warps refill it
        }
        if (S_T != nullptr) {
#pragma unroll
            for (int i = 0; i < RR; ++i) {
                float *dst = S_T + (head * DK + 8 * i + rb) * d_v + j0 + jb;
                if (!GDN2_IN_BOUNDS(kBufST, dst, 4 * CJ)) continue;
#pragma unroll
                for (int x = 0; x < CJ; ++x) dst[x] = Sr[i][x];
            }
        }
    } else {
        // ============================================================ staging
        // warp 8 + sw takes tokens sw, sw + 5, ... of a batch (MT at most); every
        // load of its tokens is issued (as 4- or 8-byte vectors) before any is used
        constexpr int MT = (TB + kStage - 1) / kStage;
        const float bscale = (PREP && fz.neg_eigval) ? 2.f : 1.f;
        const int sw = warp - 8;
        for (int k = 0; k < nb; ++k) {
            const int buf = k & 1, tb = t_begin + k * TB, nt = min(TB, len - tb);
            if (k >= 2) named_bar(BAR_EMPTY + buf, kAll);
            BfVec<CPL> rq[MT], rk[MT], rbv[MT], rl[MT];
            BfVec<JPL> rv[MT], rw[MT], rg[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const int tt = sw + kStage * m;
                if (tt < nt) {
                    const long tok = tok0 + tb + tt;
                    const long kro = (tok * H + h) * DK + CPL * lane;
                    const long vro = (tok * HV + hv) * (long)d_v + j0 + JPL * lane;
                    rq[m].load(ta.q + kro, kBufQ);
                    rk[m].load(ta.k + kro, kBufK);
                    rbv[m].load(ta.b + kro, kBufB);
                    rl[m].load(la + kro, kBufLA);
                    rv[m].load(ta.v + vro, kBufV);
                    rw[m].load(ta.w + vro, kBufW);
                    if constexpr (EPI) rg[m].load(static_cast<const __nv_bfloat16 *>(fz.gate) + vro, kBufGate);
                }
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const int tt = sw + kStage * m;
                if (tt >= nt) continue;   // warp-uniform
                float qv[CPL], kv[CPL], bv[CPL];
#pragma unroll
                for (int e = 0; e < CPL; ++e) {
                    qv[e] = rq[m].get(e);
                    kv[e] = rk[m].get(e);
                    bv[e] = rbv[m].get(e);
                }
                if constexpr (PREP) {   // q, k L2-normalised over d_k; b = sigmoid (x2 with neg_eigval)
                    float sq = 0.f, sk = 0.f;
#pragma unroll
                    for (int e = 0; e < CPL; ++e) {
                        sq = fmaf(qv[e], qv[e], sq);
                        sk = fmaf(kv[e], kv[e], sk);
                    }
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) {
                        sq += __shfl_xor_sync(0xffffffffu, sq, off);
                        sk += __shfl_xor_sync(0xffffffffu, sk, off);
                    }
                    const float iq = l2_inv(sq, fz.l2_eps), ik = l2_inv(sk, fz.l2_eps);
#pragma unroll
                    for (int e = 0; e < CPL; ++e) {
                        qv[e] *= iq;
                        kv[e] *= ik;
                        bv[e] = bscale * sigmoid_f32(bv[e]);
                    }
                }
                float dot = 0.f;
                float4 *rdst = rowd + (buf * TB + tt) * DK + CPL * lane;
#pragma unroll
                for (int e = 0; e < CPL; ++e) {
                    const float a = __expf(rl[m].get(e));
                    dot = fmaf(qv[e], kv[e], dot);
                    rdst[e] = make_float4(a, bv[e] * kv[e] * a, qv[e] * a, kv[e]);
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
                if (lane == 0) qkb[buf * TB + tt] = dot;
                float2 *cdst = cold + (buf * TB + tt) * NV + JPL * lane;
#pragma unroll
                for (int e = 0; e < JPL; ++e) {
                    const float wv = rw[m].get(e), vv = rv[m].get(e);
                    cdst[e] = make_float2((PREP ? sigmoid_f32(wv) : wv) * vv, EPI ? rg[m].get(e) : 0.f);
                }
            }
            named_bar_arrive(BAR_FULL + buf, kAll);
        }
    }
}

// Token tail of the QED variant: the same hand-off as tc_token_tail, with the
// rank-2 step of the second erase direction,
//     u = (q - (q.k / k.k) k) / sqrt(|.|^2 + eps),
//     r1_j = sum_c (b k alpha)_c S_cj,  r2_j = sum_c (c u alpha)_c S_cj,  p_j = sum_c (q alpha)_c S_cj,
//     x_j = w_j v_j - r1_j,  S_cj <- alpha_c S_cj + k_c x_j - u_c r2_j,
//     o_j = p_j + (q . k) x_j - (q . u) r2_j.
// Layout and hand-off as tc_token_tail; value heads equal key heads.
template <int DK, int NV>
__device__ __noinline__ void tc_token_tail_qed(uint8_t *smem, const TailArgs ta, const __nv_bfloat16 *__restrict__ la,
                                               __nv_bfloat16 *__restrict__ o, float *__restrict__ S_T, long tok0,
                                               int t_begin, int len, int h, int H, int j0, int d_v, long head) {
    constexpr int TB = 16, LS = NV + 4;
    constexpr int RR = DK / 8, CJ = NV / 32;
    constexpr int CPL = DK / 32, JPL = NV / 32;
    constexpr int kStage = 5, kAll = kTcThreads;
    constexpr int BAR_FULL = 5, BAR_EMPTY = 7;
    const float *sS = reinterpret_cast<const float *>(smem);
    float4 *rowd = reinterpret_cast<float4 *>(smem + DK * LS * 4);     // [2][TB][DK]: alpha, b k alpha, q alpha, k
    float2 *rowe = reinterpret_cast<float2 *>(rowd + 2 * TB * DK);      // [2][TB][DK]: c u alpha, u
    float *cold = reinterpret_cast<float *>(rowe + 2 * TB * DK);         // [2][TB][NV]: w v
    float2 *qkb = reinterpret_cast<float2 *>(cold + 2 * TB * NV);        // [2][TB]: q . k, q . u
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nb = (len - t_begin + TB - 1) / TB;
    if (warp < 8) {
        const int rb = lane & 7, cb = lane >> 3, jb = (4 * warp + cb) * CJ;
        float Sr[RR][CJ];
#pragma unroll
        for (int i = 0; i < RR; ++i)
#pragma unroll
            for (int x = 0; x < CJ; ++x) Sr[i][x] = sS[(8 * i + rb) * LS + jb + x];
        for (int k = 0; k < nb; ++k) {
            const int buf = k & 1, tb = t_begin + k * TB, nt = min(TB, len - tb);
            named_bar(BAR_FULL + buf, kAll);
            for (int tt = 0; tt < nt; ++tt) {
                const float4 *rd = rowd + (buf * TB + tt) * DK;
                const float2 *re = rowe + (buf * TB + tt) * DK;
                float r1[CJ], r2[CJ], pq[CJ];
#pragma unroll
                for (int x = 0; x < CJ; ++x) r1[x] = r2[x] = pq[x] = 0.f;
#pragma unroll
                for (int i = 0; i < RR; ++i) {
                    const float4 xr = rd[8 * i + rb];
                    const float2 xe = re[8 * i + rb];
#pragma unroll
                    for (int x = 0; x < CJ; ++x) {
                        r1[x] = fmaf(xr.y, Sr[i][x], r1[x]);
                        r2[x] = fmaf(xe.x, Sr[i][x], r2[x]);
                        pq[x] = fmaf(xr.z, Sr[i][x], pq[x]);
                    }
                }
#pragma unroll
                for (int off = 1; off < 8; off <<= 1)
#pragma unroll
                    for (int x = 0; x < CJ; ++x) {
                        r1[x] += __shfl_xor_sync(0xffffffffu, r1[x], off);
                        r2[x] += __shfl_xor_sync(0xffffffffu, r2[x], off);
                        pq[x] += __shfl_xor_sync(0xffffffffu, pq[x], off);
                    }
                const float2 qs = qkb[buf * TB + tt];
                float x1[CJ], ov[CJ];
#pragma unroll
                for (int x = 0; x < CJ; ++x) {
                    x1[x] = cold[(buf * TB + tt) * NV + jb + x] - r1[x];
                    ov[x] = fmaf(qs.x, x1[x], fmaf(-qs.y, r2[x], pq[x]));
                }
#pragma unroll
                for (int i = 0; i < RR; ++i) {
                    const float4 xr = rd[8 * i + rb];
                    const float2 xe = re[8 * i + rb];
#pragma unroll
                    for (int x = 0; x < CJ; ++x)
                        Sr[i][x] = fmaf(xr.x, Sr[i][x], fmaf(xr.w, x1[x], -xe.y * r2[x]));
                }
                if (rb == 0) {
                    __nv_bfloat16 *dst = o + ((tok0 + tb + tt) * H + h) * (long)d_v + j0 + jb;
                    if (GDN2_IN_BOUNDS(kBufO, dst, 2 * CJ)) {
#pragma unroll
                        for (int x = 0; x < CJ; x += 2)
                            *reinterpret_cast<uint32_t *>(dst + x) = pack_bf16x2(ov[x], ov[x + 1]);
                    }
                }
            }
            if (k + 2 < nb) named_bar_arrive(BAR_EMPTY + buf, kAll);
        }
        if (S_T != nullptr) {
#pragma unroll
            for (int i = 0; i < RR; ++i) {
                float *dst = S_T + (head * DK + 8 * i + rb) * d_v + j0 + jb;
                if (!GDN2_IN_BOUNDS(kBufST, dst, 4 * CJ)) continue;
#pragma unroll
                for (int x = 0; x < CJ; ++x) dst[x] = Sr[i][x];
            }
        }
    } else {
        constexpr int MT = (TB + kStage - 1) / kStage;
        const int sw = warp - 8;
        for (int k = 0; k < nb; ++k) {
            const int buf = k & 1, tb = t_begin + k * TB, nt = min(TB, len - tb);
            if (k >= 2) named_bar(BAR_EMPTY + buf, kAll);
            BfVec<CPL> rq[MT], rk[MT], rbv[MT], rc[MT], rl[MT];
            BfVec<JPL> rv[MT], rw[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const int tt = sw + kStage * m;
                if (tt < nt) {
                    const long tok = tok0 + tb + tt;
                    const long kro = (tok * H + h) * DK + CPL * lane;
                    const long vro = (tok * H + h) * (long)d_v + j0 + JPL * lane;
                    rq[m].load(ta.q + kro, kBufQ);
                    rk[m].load(ta.k + kro, kBufK);
                    rbv[m].load(ta.b + kro, kBufB);
                    rc[m].load(ta.c + kro, kBufC);
                    rl[m].load(la + kro, kBufLA);
                    rv[m].load(ta.v + vro, kBufV);
                    rw[m].load(ta.w + vro, kBufW);
                }
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const int tt = sw + kStage * m;
                if (tt >= nt) continue;   // warp-uniform
                float qv[CPL], kv[CPL];
                float qk = 0.f, kk = 0.f;
#pragma unroll
                for (int e = 0; e < CPL; ++e) {
                    qv[e] = rq[m].get(e);
                    kv[e] = rk[m].get(e);
                    qk = fmaf(qv[e], kv[e], qk);
                    kk = fmaf(kv[e], kv[e], kk);
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    qk += __shfl_xor_sync(0xffffffffu, qk, off);
                    kk += __shfl_xor_sync(0xffffffffu, kk, off);
                }
                const float coef = kk > 0.f ? qk / kk : 0.f;
                float rr = 0.f;
#pragma unroll
                for (int e = 0; e < CPL; ++e) {
                    const float r = qv[e] - coef * kv[e];
                    rr = fmaf(r, r, rr);
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) rr += __shfl_xor_sync(0xffffffffu, rr, off);
                const float den = rr + ta.qed_eps, nu = den > 0.f ? rsqrtf(den) : 0.f;
                float qu = 0.f;
                float4 *rdst = rowd + (buf * TB + tt) * DK + CPL * lane;
                float2 *edst = rowe + (buf * TB + tt) * DK + CPL * lane;
#pragma unroll
                for (int e = 0; e < CPL; ++e) {
                    const float a = __expf(rl[m].get(e));
                    const float u = (qv[e] - coef * kv[e]) * nu;
                    qu = fmaf(qv[e], u, qu);
                    rdst[e] = make_float4(a, rbv[m].get(e) * kv[e] * a, qv[e] * a, kv[e]);
                    edst[e] = make_float2(rc[m].get(e) * u * a, u);
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) qu += __shfl_xor_sync(0xffffffffu, qu, off);
                if (lane == 0) qkb[buf * TB + tt] = make_float2(qk, qu);
                float *cdst = cold + (buf * TB + tt) * NV + JPL * lane;
#pragma unroll
                for (int e = 0; e < JPL; ++e) cdst[e] = rw[m].get(e) * rv[m].get(e);
            }
            named_bar_arrive(BAR_FULL + buf, kAll);
        }
    }
}

// PREP fuses the input prep (raw q, k, b, w); EPI the gated RMS norm of each
// output row before it is stored (d_v == NV: one CTA holds the whole row).
template <int DK, int NV, bool PREP = false, bool EPI = false, bool VARLEN = false, bool QED = false>
__global__ void __launch_bounds__(kTcThreads, 1)
chunk_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_o,
                    const __grid_constant__ CUtensorMap tm_c,
                    const __nv_bfloat16 *__restrict__ la,
                    const float *__restrict__ S0,
                    __nv_bfloat16 *__restrict__ o, float *__restrict__ S_T, int T, int H, int HV, int d_v,
                    const int *__restrict__ cu_seqlens, unsigned long long wait_ns, const FuseArgs fz,
                    const TailArgs ta) {
    static_assert(!EPI || NV <= 128, "epilogue weight slice");
    static_assert(!QED || (!PREP && !EPI && !VARLEN), "the QED variant has no fusion and no packing");
    using Cfg = TcCfg<DK, NV>;
    // tokens per chunk: 64, or 32 with the query direction (two pseudo-rows each)
    constexpr int CH = QED ? 32 : 64;
    constexpr uint32_t KEY_BYTES = CH * DK * 2u, VAL_BYTES = CH * NV * 2u;   // one tensor, one chunk (TMA)
    // packed bf16x2 operand products in the prep, except where an output epilogue
    // normalises each row (it turns the extra rounding of small rows into a large
    // relative error) or the input prep rescales the rows
    constexpr bool kPackedPrep = !PREP && !EPI;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    const uint32_t sb = smem_u32(smem);

    const int tid = threadIdx.x, warp = tid >> 5;
    // CTA: value head hv (of HV) reading key head h = hv / (HV / H), sequence bb.
    // A sequence is tokens [tok0, tok0 + len): bb * T + [0, T) for equal-length
    // batches, [cu[bb], cu[bb + 1]) when packed (the TMA maps then have one
    // "batch" of all tokens: coordinates (c, head, tok0 + 64 n, 0)).
    const int j0 = blockIdx.x * NV, hv = blockIdx.y;
    int bb = blockIdx.z;
    if constexpr (VARLEN) bb = longest_first_sequence(cu_seqlens, gridDim.z, bb, reinterpret_cast<int *>(smem));
    const int h = hv / (HV / H);
    long tok0 = (long)bb * T;
    int len = T, tma_t0 = 0, tma_b = bb;
    if constexpr (VARLEN) {
        const bool cu_ok = GDN2_IN_BOUNDS(kBufCU, cu_seqlens + bb, 8);
        const int a = cu_ok ? cu_seqlens[bb] : -1, e = cu_ok ? cu_seqlens[bb + 1] : -1;
        if (a < 0 || e < a || e > T) {   // malformed packing: this sequence is skipped
            if (threadIdx.x == 0) record_status(kStatusBadArgs);
            return;
        }
        tok0 = a;
        len = e - a;
        tma_t0 = a;
        tma_b = 0;
    }
    const int NC = (len + CH - 1) / CH;   // the last chunk may be partial
    const long head = (long)bb * HV + hv;

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
    uint64_t *qb_full = bars + 0;     // [2] TMA q, b of a chunk landed (stage m % 2)
    uint64_t *k_full = bars + 2;      // [3] TMA k of a chunk landed (stage m % 3)
    uint64_t *v_full = bars + 5;      // TMA v landed
    uint64_t *w_full = bars + 6;      // TMA w landed
    uint64_t *v_free = bars + 7;      // MMA3 complete: the v tile (W.V) is free (tcgen05.commit)
    uint64_t *w_free = bars + 8;      // key done with the w tile (W.V formed, solve scratch released)
    uint64_t *full = bars + 9;        // [2] key products of a chunk ready
    uint64_t *empty_qe = bars + 11;   // [2] chain's MMA_T done: Q~/E (then -E S) tiles of the stage free
    uint64_t *empty_k = bars + 13;    // [3] chain's MMA_u done: K~ tile of the stage free
    uint64_t *empty_pg = bars + 16;   // [2] chain done with P of the stage
    uint64_t *utfree = bars + 18;     // chain has read U out of TMEM
    uint64_t *bk1 = bars + 19;        // MMA1 complete
    uint64_t *bct = bars + 20;        // MMA_T complete (chain)
    uint64_t *bc1 = bars + 21, *bc2 = bars + 22, *bc3 = bars + 23;
    uint64_t *drain = bars + 24;      // [2] teardown: key and chain MMA issuers (the MMA3 issuer: drain3)
    uint64_t *ut_ready = bars + 26;   // MMA3 of a chunk complete: T(W.V) in TMEM
    uint64_t *t_free = bars + 27;     // MMA_T complete: the T tile is free for the next solve
    uint64_t *drain3 = bars + 28;     // teardown: the MMA3 issuer (key thread 128)
    constexpr int kNumBars = 29;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + Cfg::OFF_TMEMP);
    float *gC = reinterpret_cast<float *>(smem + Cfg::OFF_GC);
    float *sA = reinterpret_cast<float *>(smem + Cfg::OFF_SCR);

    // ---------------------------------------------------------------- setup
    for (uint32_t off = tid * 16u; off < Cfg::OFF_CARRY; off += kTcThreads * 16u) st_shared_v4(sb + off, 0u, 0u, 0u, 0u);
    for (int i = tid; i < 3 * 256; i += kTcThreads) gC[i] = 1.f;   // channels >= d_k keep factors of 1
    volatile int *stop_at = reinterpret_cast<volatile int *>(smem + Cfg::OFF_STOP);
    if (tid == 0) {
        *stop_at = 0x7fffffff;
        // kept for the teardown, so that no register holds them through the main loop
        *reinterpret_cast<long *>(smem + Cfg::OFF_SEQ) = tok0;
        reinterpret_cast<int *>(smem + Cfg::OFF_SEQ)[2] = len;
        reinterpret_cast<int *>(smem + Cfg::OFF_SEQ)[3] = bb;
    }
    if constexpr (EPI) {
        float *nw = reinterpret_cast<float *>(smem + Cfg::OFF_NW);
        for (int i = tid; i < NV; i += kTcThreads)
            nw[i] = GDN2_IN_BOUNDS(kBufNW, fz.norm_weight + j0 + i, 4) ? fz.norm_weight[j0 + i] : 0.f;
    }
    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i) mbar_init(bars + i, 1);
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
                const int r = tma_t0 + n * CH;
                for (int kb = 0; kb < DK / 64; ++kb) {
                    tma_prefetch_l2_4d(&tm_q, kb * 64, h, r, tma_b);
                    tma_prefetch_l2_4d(&tm_k, kb * 64, h, r, tma_b);
                    tma_prefetch_l2_4d(&tm_b, kb * 64, h, r, tma_b);
                    if constexpr (QED) tma_prefetch_l2_4d(&tm_c, kb * 64, h, r, tma_b);
                }
                for (int vb = 0; vb < Cfg::VB; ++vb) {
                    tma_prefetch_l2_4d(&tm_v, j0 + vb * 64, hv, r, tma_b);
                    tma_prefetch_l2_4d(&tm_w, j0 + vb * 64, hv, r, tma_b);
                }
            };
            // chunks requested into L2 ahead of their loads: one for the plain kernel,
            // where a deeper prefetch competes with the demand loads; three with the
            // fused prep or epilogue, whose longer chunk period leaves room for it
            constexpr int kPrefetch = (PREP || EPI) ? 3 : 1;
            for (int p = 0; p < kPrefetch && p < NC; ++p) prefetch(p);
            int nq = 0, nk = 0, nw = 0, nv = 0;   // next chunk to load for each group
            int lim = NC;                         // chunks from a handed-off one on are not loaded
            uint64_t t0 = globaltimer_ns();
            while (nq < lim || nk < lim || nw < lim || nv < lim) {
                bool progress = false;
                if (nq < lim && (nq < 2 || mbar_test_wait(&empty_qe[nq & 1], static_cast<uint32_t>(((nq >> 1) - 1) & 1)))) {
                    const int s = nq & 1, r = tma_t0 + nq * CH;
                    const uint32_t oqe = s ? Cfg::OFF_QE1 : Cfg::OFF_QE0;
                    mbar_arrive_expect_tx(&qb_full[s], (QED ? 3u : 2u) * KEY_BYTES);
                    for (int kb = 0; kb < DK / 64; ++kb) {
                        tma_load_4d(smem + oqe + kb * 16384, &tm_q, &qb_full[s], kb * 64, h, r, tma_b);
                        if constexpr (QED) {   // c into Q~ rows 32-63, b into E rows 32-63
                            tma_load_4d(smem + oqe + kb * 16384 + 4096, &tm_c, &qb_full[s], kb * 64, h, r, tma_b);
                            tma_load_4d(smem + oqe + kb * 16384 + 8192 + 4096, &tm_b, &qb_full[s], kb * 64, h, r,
                                        tma_b);
                        } else {
                            tma_load_4d(smem + oqe + kb * 16384 + 8192, &tm_b, &qb_full[s], kb * 64, h, r, tma_b);
                        }
                    }
                    if (nq + kPrefetch < NC) prefetch(nq + kPrefetch);
                    ++nq;
                    progress = true;
                }
                if (nk < lim && (nk < 3 || mbar_test_wait(&empty_k[nk % 3], static_cast<uint32_t>((nk / 3 - 1) & 1)))) {
                    const int s3 = nk % 3, r = tma_t0 + nk * CH;
                    mbar_arrive_expect_tx(&k_full[s3], KEY_BYTES);
                    for (int kb = 0; kb < DK / 64; ++kb)   // QED: k into K~ rows 32-63
                        tma_load_4d(smem + Cfg::OFF_K + s3 * 16384 + kb * 8192 + (QED ? 4096 : 0), &tm_k, &k_full[s3],
                                    kb * 64, h, r, tma_b);
                    ++nk;
                    progress = true;
                }
                if (nw < lim && (nw < 1 || mbar_test_wait(w_free, static_cast<uint32_t>((nw - 1) & 1)))) {
                    const int r = tma_t0 + nw * CH;
                    mbar_arrive_expect_tx(w_full, VAL_BYTES);
                    for (int vb = 0; vb < Cfg::VB; ++vb)
                        tma_load_4d(smem + Cfg::OFF_W + vb * 8192, &tm_w, w_full, j0 + vb * 64, hv, r, tma_b);
                    ++nw;
                    progress = true;
                }
                if (nv < lim && (nv < 1 || mbar_test_wait(v_free, static_cast<uint32_t>((nv - 1) & 1)))) {
                    const int r = tma_t0 + nv * CH;
                    mbar_arrive_expect_tx(v_full, VAL_BYTES);
                    for (int vb = 0; vb < Cfg::VB; ++vb)   // QED: v into rows 32-63
                        tma_load_4d(smem + Cfg::OFF_V + vb * 8192 + (QED ? 4096 : 0), &tm_v, v_full, j0 + vb * 64, hv,
                                    r, tma_b);
                    ++nv;
                    progress = true;
                }
                lim = min(NC, *stop_at);
                const uint64_t now = globaltimer_ns();
                if (progress) t0 = now;
                else if (now - t0 > wait_ns) { failed = true; break; }
            }
            if (failed || lim < NC) {
                // handed off, or stopped by a failed wait: let every issued load land
                // (each wait bounded) before the shared memory is reused or released
                // (the last load of each barrier slot completes that slot's last phase)
                bool ok = true;
                for (int j = max(0, nq - 2); j < nq; ++j)
                    ok &= mbar_wait(&qb_full[j & 1], static_cast<uint32_t>((j >> 1) & 1), wait_ns);
                for (int j = max(0, nk - 3); j < nk; ++j)
                    ok &= mbar_wait(&k_full[j % 3], static_cast<uint32_t>((j / 3) & 1), wait_ns);
                if (nv > 0) ok &= mbar_wait(v_full, static_cast<uint32_t>((nv - 1) & 1), wait_ns);
                if (nw > 0) ok &= mbar_wait(w_full, static_cast<uint32_t>((nw - 1) & 1), wait_ns);
                if (!ok) failed = true;
            }
        }
    } else if (tid < kKeyThreads) {
        // ============================================================ key side
        // Two-stage pipeline over chunks: while warps 0-3 (group A) invert
        // I + A of chunk m, warps 4-7 (group B) prepare chunk m+1; everything
        // else is done by all eight warps.
        const int t = tid, l = tid & 31, kq = warp & 3, kh = warp >> 2;   // lane quarter, column half
        const bool grp_b = t >= 128;
        uint32_t ph1 = 0;
        // MMA1 is issued by key thread 0 and MMA3 by key thread 128 (warp 4), so that
        // the two issues, each held while the tensor pipe works through its queue,
        // overlap at the turn of an iteration instead of following each other
        constexpr int kMma3Issuer = 128;
        bool mma3_failed = false;   // thread kMma3Issuer only
        float *carry = reinterpret_cast<float *>(smem + Cfg::OFF_CARRY);
        float2 *nrm = reinterpret_cast<float2 *>(smem + Cfg::OFF_NRM);
        // group B: log_alpha of the next chunk to prepare
        typename std::conditional<QED, PrepLAQ<DK>, PrepLA<DK>>::type lan;
        // prep of chunk n (stage sn of the Q~/E tiles, stage s3n of K~) by group B
        auto prep = [&](int n, uint32_t oqe, uint32_t okt) {
            if constexpr (QED)
                prep_chunk_qed<DK>(smem, oqe, okt, lan, gC + (n % 3) * 256, nrm, t - 128, 4, n, stop_at, ta.qed_eps);
            else
                prep_chunk<DK, PREP, VARLEN, kPackedPrep>(smem, oqe, okt, lan, gC + (n % 3) * 256, carry, t - 128, 4,
                                                          n, stop_at, fz, nrm, min(64, len - n * 64));
        };
        // prologue: prep of chunk 0 (group B)
        if (NC > 0) {
            if (grp_b) lan.load(la, tok0, 0, h, len, H, t - 128);
            bool ok = mbar_wait(&qb_full[0], 0u, wait_ns);
            ok = ok && mbar_wait(&k_full[0], 0u, wait_ns);
            if (group_any(1, kKeyThreads, !ok)) failed = true;
            else if (grp_b) prep(0, Cfg::OFF_QE0, Cfg::OFF_K);
        }
        for (int m = 0; m < NC && !failed; ++m) {
            const int s = m & 1;
            const uint32_t OQE = s ? Cfg::OFF_QE1 : Cfg::OFF_QE0, OK = Cfg::OFF_K + (m % 3) * 16384u;
            const uint32_t OP = s ? Cfg::OFF_P1 : Cfg::OFF_P0;
            // prep of chunk m is complete: chunk 0 here, later chunks before the
            // barriers that close the previous iteration
            if (m == 0) named_bar(1, kKeyThreads);
            if (*stop_at <= m) {   // chunk m and the rest of the sequence go to the token tail
                if (t == 0) mbar_arrive(&full[s]);   // the chain stops at the same chunk
                break;
            }
            // log_alpha of chunk m+1, a whole iteration ahead of its use
            if (grp_b && m + 1 < NC) lan.load(la, tok0, m + 1, h, len, H, t - 128);
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
            // W.V in place in the v tile while MMA1 runs (the solve scratch overlaps
            // the w tile, so this comes first)
            {
                bool ok = mbar_wait(v_full, static_cast<uint32_t>(m & 1), wait_ns);
                ok = ok && mbar_wait(w_full, static_cast<uint32_t>(m & 1), wait_ns);
                if (group_any(1, kKeyThreads, !ok)) { failed = true; break; }
                if constexpr (QED) {
                    // 32 tokens of v (rows 32-63) and w (rows 0-31) -> pseudo-rows 2t = w.v,
                    // 2t + 1 = 0: every raw row is read before any expanded row is written
                    constexpr int CPR = NV / 8, PPT = 32 * CPR / kKeyThreads;   // 16-byte chunks
                    uint4 wv[PPT];
#pragma unroll
                    for (int i = 0; i < PPT; ++i) {
                        const int idx = t + i * kKeyThreads, tok = idx / CPR, ch = idx % CPR;
                        const uint32_t sub = (ch >> 3) * 8192u;
                        uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
                        ld_shared_v4(sb + Cfg::OFF_V + sub + sw128_chunk(32 + tok, ch & 7), a0, a1, a2, a3);
                        ld_shared_v4(sb + Cfg::OFF_W + sub + sw128_chunk(tok, ch & 7), b0, b1, b2, b3);
                        wv[i] = mul_bf16x8(make_uint4(a0, a1, a2, a3), make_uint4(b0, b1, b2, b3));
                    }
                    named_bar(1, kKeyThreads);
#pragma unroll
                    for (int i = 0; i < PPT; ++i) {
                        const int idx = t + i * kKeyThreads, tok = idx / CPR, ch = idx % CPR;
                        const uint32_t sub = (ch >> 3) * 8192u;
                        st_shared_v4(sb + Cfg::OFF_V + sub + sw128_chunk(2 * tok, ch & 7), wv[i].x, wv[i].y, wv[i].z,
                                     wv[i].w);
                        st_shared_v4(sb + Cfg::OFF_V + sub + sw128_chunk(2 * tok + 1, ch & 7), 0u, 0u, 0u, 0u);
                    }
                }
#pragma unroll
                for (int it = 0; it < (QED ? 0 : Cfg::VAL_TILE / 16 / kKeyThreads); ++it) {
                    const uint32_t off = (t + it * kKeyThreads) * 16u;
                    uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
                    ld_shared_v4(sb + Cfg::OFF_V + off, a0, a1, a2, a3);
                    ld_shared_v4(sb + Cfg::OFF_W + off, b0, b1, b2, b3);
                    uint4 r4;
                    if (PREP) {   // w arrives raw: sigmoid(w) . v, rounded once
                        const uint32_t vv[4] = {a0, a1, a2, a3}, ww[4] = {b0, b1, b2, b3};
                        uint32_t rr[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 hx = mul_f32x2(make_float2(bf16_lo(ww[e]), bf16_hi(ww[e])), make_float2(0.5f, 0.5f));
                            float2 th;
                            asm("tanh.approx.f32 %0, %1;" : "=f"(th.x) : "f"(hx.x));
                            asm("tanh.approx.f32 %0, %1;" : "=f"(th.y) : "f"(hx.y));
                            const float2 sg = fma_f32x2(th, make_float2(0.5f, 0.5f), make_float2(0.5f, 0.5f));
                            const float2 x = mul_f32x2(sg, make_float2(bf16_lo(vv[e]), bf16_hi(vv[e])));
                            rr[e] = pack_bf16x2(x.x, x.y);
                        }
                        r4 = make_uint4(rr[0], rr[1], rr[2], rr[3]);
                    } else {
                        r4 = mul_bf16x8(make_uint4(a0, a1, a2, a3), make_uint4(b0, b1, b2, b3));
                    }
                    // packed: the rows after the sequence end hold the next sequence's tokens
                    if (VARLEN && ((off & 8191u) >> 7) >= static_cast<uint32_t>(len - m * 64))
                        r4 = make_uint4(0u, 0u, 0u, 0u);
                    st_shared_v4(sb + Cfg::OFF_V + off, r4.x, r4.y, r4.z, r4.w);
                }
                fence_proxy_async_smem();   // MMA3 reads W.V
            }
            {
                bool ok = !mma3_failed && mbar_wait(bk1, ph1, wait_ns);
                ph1 ^= 1u;
                // P of this stage was last read by the chain two chunks ago
                if (m >= 2) ok = ok && mbar_wait(&empty_pg[s], static_cast<uint32_t>(((m >> 1) - 1) & 1), wait_ns);
                if (group_any(1, kKeyThreads, !ok)) { failed = true; break; }
            }
            tc_fence_after();
            // ------------------------------------------- read out P' and A
            // warp: lanes 32*kq.., columns 32*kh..; P' in lanes 0-63, A' in 64-127
            {
                float x[32];
                tmem_ld32(t_KT + lane_q + 32 * kh, x);
                // warp-uniform block position: columns 32 kh.. against rows 32 (kq % 2)..;
                // only the diagonal block needs per-element masks
                const int rb = kq & 1, r = 32 * rb + l;
                if constexpr (QED) {   // masks by token: pseudo-rows 2t, 2t + 1 belong to token t
                    if (kq < 2) {   // P: token row r (rows 32-63 hold no token) sees rows <= 2r + 1
#pragma unroll
                        for (int e = 0; e < 32; ++e) x[e] = (rb == 0 && 32 * kh + e <= 2 * l + 1) ? x[e] : 0.f;
                    } else {        // A: pseudo-row r sees the rows of earlier tokens only
#pragma unroll
                        for (int e = 0; e < 32; ++e) x[e] = (32 * kh + e < (r & ~1)) ? x[e] : 0.f;
                    }
                }
                if (kq < 2) {   // P = lower(Q~ K~^T), diagonal included
                    if (QED) {
                    } else if (kh > rb) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) x[e] = 0.f;
                    } else if (kh == rb) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) x[e] = e <= l ? x[e] : 0.f;
                    }
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        st_shared_v4(sb + OP + sw128_chunk(r, 4 * kh + q4), pack_bf16x2(x[8 * q4], x[8 * q4 + 1]),
                                     pack_bf16x2(x[8 * q4 + 2], x[8 * q4 + 3]), pack_bf16x2(x[8 * q4 + 4], x[8 * q4 + 5]),
                                     pack_bf16x2(x[8 * q4 + 6], x[8 * q4 + 7]));
                } else {        // A = strict_lower(E K~^T), fp32 into the solve scratch
                    if (QED) {
                    } else if (kh > rb) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) x[e] = 0.f;
                    } else if (kh == rb) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) x[e] = e < l ? x[e] : 0.f;
                    }
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        *reinterpret_cast<float4 *>(sA + r * Cfg::LDA + 32 * kh + e) = make_float4(x[e], x[e + 1], x[e + 2], x[e + 3]);
                }
            }
            tc_fence_before();
            named_bar(1, kKeyThreads);
            // ------------- group A: T = (I + A)^{-1};  group B: prep of chunk m+1
            bool ok_b = true;
            if (!grp_b) {
                // the chain's MMA_T has read T of the previous chunk
                if (m >= 1) ok_b = mbar_wait(t_free, static_cast<uint32_t>((m - 1) & 1), wait_ns);
                ok_b = !group_any(3, 128, !ok_b);
                if (ok_b) unit_lower_inverse64<Cfg::LDA>(sA, smem + Cfg::OFF_T, t, 3);
            } else if (m + 1 < NC) {
                const int sn = (m + 1) & 1, s3n = (m + 1) % 3;
                ok_b = mbar_wait(&qb_full[sn], static_cast<uint32_t>(((m + 1) >> 1) & 1), wait_ns);
                ok_b = ok_b && mbar_wait(&k_full[s3n], static_cast<uint32_t>(((m + 1) / 3) & 1), wait_ns);
                ok_b = !group_any(4, 128, !ok_b);
                if (ok_b) prep(m + 1, sn ? Cfg::OFF_QE1 : Cfg::OFF_QE0, Cfg::OFF_K + s3n * 16384u);
            }
            // P (warps 0, 1, 4, 5), T and the prepared tiles are written: hand the
            // chunk to the chain, then MMA3 [. ; T] (W.V) -> T (W.V) in TMEM, whose
            // commits free the v tile and tell the chain; only the issuer waits
            // for the chain to have read the previous U out of TMEM
            fence_proxy_async_smem();
            if (group_any(1, kKeyThreads, !ok_b)) { failed = true; break; }
            if (t == 0) {
                mbar_arrive(w_free);   // w tile (solve scratch) is free
                mbar_arrive(&full[s]);
            }
            if (t == kMma3Issuer) {
                const bool ok_ut = (m == 0) || mbar_wait(utfree, static_cast<uint32_t>((m - 1) & 1), wait_ns);
                if (ok_ut) {
                    tc_fence_after();
                    const uint32_t id3 = idesc_bf16(128, NV, false, true);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        umma_bf16(t_UT, sdesc_sw128(sb + Cfg::OFF_T - 8192 + ks * 32, 16, 1024),
                                  sdesc_sw128(sb + Cfg::OFF_V + ks * 2048, 8192, 1024), id3, ks > 0 ? 1u : 0u);
                    umma_commit(v_free);
                    umma_commit(ut_ready);
                } else {
                    mma3_failed = true;   // the key group stops at the next MMA1 wait
                }
            }
        }
        if (mma3_failed) failed = true;
        if (t == 0 || t == kMma3Issuer) {   // wait (bounded) for each issuer's MMAs before teardown
            uint64_t *db = (t == 0) ? &drain[0] : drain3;
            umma_commit(db);
            mbar_wait(db, 0u, wait_ns);
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
                if (S0 != nullptr && c < DK &&
                    GDN2_IN_BOUNDS(kBufS0, S0 + (head * DK + c) * d_v + j0 + jc * 32, 128)) {
                    const float4 *src = reinterpret_cast<const float4 *>(S0 + (head * DK + c) * d_v + j0 + jc * 32);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float4 x = src[e];
                        sv[4 * e] = x.x; sv[4 * e + 1] = x.y; sv[4 * e + 2] = x.z; sv[4 * e + 3] = x.w;
                    }
                }
                tmem_st32(t_S + lane_q + jc * 32, sv);
                if (NC == 0 && S_T != nullptr && c < DK &&   // empty sequence: S_T = S0
                    GDN2_IN_BOUNDS(kBufST, S_T + (head * DK + c) * d_v + j0 + jc * 32, 128)) {
                    float4 *dst = reinterpret_cast<float4 *>(S_T + (head * DK + c) * d_v + j0 + jc * 32);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        dst[e] = make_float4(sv[4 * e], sv[4 * e + 1], sv[4 * e + 2], sv[4 * e + 3]);
                }
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
        if (NC > 0 && S0 != nullptr) {
            // the chain carries the state scaled by 2^ref of the chunk it enters: S0
            // takes chunk 0's factor once chunk 0 is prepared (later chunks get theirs
            // with the state update); the loop's own wait on full[0] then passes at once
            const bool ok = mbar_wait(&full[0], 0u, wait_ns);
            if (group_any(2, kChainThreads, !ok)) failed = true;
            else if (*stop_at > 0) {
                const int c = t;
                const float f = gC[128 + c];
#pragma unroll 1
                for (int jc = 0; jc < NV / 32; ++jc) {
                    float sv[32];
                    tmem_ld32(t_S + lane_q + jc * 32, sv);
#pragma unroll
                    for (int e = 0; e < 32; ++e) sv[e] *= f;
                    tmem_st32(t_S + lane_q + jc * 32, sv);
                    if (c < DK) {
                        const uint32_t tile = sb + Cfg::OFF_S + ((jc * 32) >> 6) * 16384u;
                        const uint32_t ch0 = ((jc * 32) & 63) >> 3;
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4)
                            st_shared_v4(tile + sw128_chunk(c, ch0 + q4), pack_bf16x2(sv[8 * q4], sv[8 * q4 + 1]),
                                         pack_bf16x2(sv[8 * q4 + 2], sv[8 * q4 + 3]),
                                         pack_bf16x2(sv[8 * q4 + 4], sv[8 * q4 + 5]),
                                         pack_bf16x2(sv[8 * q4 + 6], sv[8 * q4 + 7]));
                    }
                }
                tmem_st_wait();
                fence_proxy_async_smem();
                tc_fence_before();
                named_bar(2, kChainThreads);
            }
        }
        uint32_t ph1 = 0, ph2 = 0, ph3 = 0, pht = 0;
        for (int n = 0; n < NC && !failed; ++n) {
            const int s = n & 1;
            if constexpr (EPI) {   // the epilogue's gate tile, into L2 a whole chain pass ahead
                const int r = t >> 1;   // two threads per row: 2 x 128-byte lines of the NV slice
                if (n * 64 + r < len && (t & 1) * 64 < NV)
                    prefetch_l2(static_cast<const __nv_bfloat16 *>(fz.gate) +
                                ((tok0 + (long)n * 64 + r) * HV + hv) * (long)d_v + j0 + (t & 1) * 64);
            }
            const uint32_t OQE = s ? Cfg::OFF_QE1 : Cfg::OFF_QE0, OK = Cfg::OFF_K + (n % 3) * 16384u;
            const uint32_t OP = s ? Cfg::OFF_P1 : Cfg::OFF_P0;
            // MMA_s needs only chunk n's prepared Q~ and E (done before the hand-off of
            // chunk n - 1, or, for chunk 0, before full[0]) and the chain's own state,
            // so it is issued before the wait for the rest of chunk n's key products
            // (T, P and the next chunk's prep); for the same reason chunk n's own stop
            // decision is final here
            if (n == 0) {
                const bool ok = mbar_wait(&full[s], static_cast<uint32_t>((n >> 1) & 1), wait_ns);
                if (group_any(2, kChainThreads, !ok)) { failed = true; break; }
            }
            if (*stop_at <= n) break;   // handed to the token tail from chunk n on
            // ------------------------------------------------------ MMA_s
            if (t == 0) {
                tc_fence_after();
                const uint32_t ids = idesc_bf16(128, NV, false, true);
#pragma unroll
                for (int ks = 0; ks < DK / 16; ++ks)
                    umma_bf16(t_X, sdesc_sw128(sb + OQE + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
                              sdesc_sw128(sb + Cfg::OFF_S + ks * 2048, 16384, 1024), ids, ks > 0 ? 1u : 0u);
                umma_commit(bc1);
                if (!EPI) bulk_wait_read_all();   // the previous O store has read the U tile
            }
            if (n > 0) {
                const bool ok = mbar_wait(&full[s], static_cast<uint32_t>((n >> 1) & 1), wait_ns);
                if (group_any(2, kChainThreads, !ok)) { failed = true; break; }
            }
            const int stop_now = *stop_at;   // includes chunk n + 1's decision (its prep is done)
            {
                const bool ok = mbar_wait(bc1, ph1, wait_ns);
                ph1 ^= 1u;
                if (group_any(2, kChainThreads, !ok)) { failed = true; break; }
            }
            tc_fence_after();
            // -E S (TMEM lanes 64-127 of X) -> bf16 over the E tiles of this stage
            // (DK = 64: over Q~ and E), dead since MMA_s: the B operand of MMA_T
            if ((warp & 3) >= 2) {
                const int r = t - 64;
#pragma unroll 1
                for (int jc = 0; jc < NV / 32; ++jc) {
                    float x[32];
                    tmem_ld32(t_X + lane_q + jc * 32, x);
                    const uint32_t tile = sb + OQE + Cfg::es_tile((jc * 32) >> 6);
                    const uint32_t ch0 = ((jc * 32) & 63) >> 3;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const int e = 8 * q4;
                        st_shared_v4(tile + sw128_chunk(r, ch0 + q4), pack_bf16x2(-x[e], -x[e + 1]),
                                     pack_bf16x2(-x[e + 2], -x[e + 3]), pack_bf16x2(-x[e + 4], -x[e + 5]),
                                     pack_bf16x2(-x[e + 6], -x[e + 7]));
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar(2, kChainThreads);
            // ------------------------------------------------------ MMA_T
            // [. ; T] (-E S) accumulated onto MMA3's T (W.V): rows 64-127 = U; its
            // commits free the T tile (next solve) and the Q~/E stage (producer)
            bool ut_fail = false;
            if (t == 0) {
                ut_fail = !mbar_wait(ut_ready, static_cast<uint32_t>(n & 1), wait_ns);   // T(W.V) of this chunk
                if (!ut_fail) {
                    tc_fence_after();
                    const uint32_t idt = idesc_bf16(128, NV, false, true);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        umma_bf16(t_UT, sdesc_sw128(sb + Cfg::OFF_T - 8192 + ks * 32, 16, 1024),
                                  sdesc_sw128(sb + OQE + Cfg::es_tile(0) + ks * 2048, Cfg::ES_LBO, 1024), idt, 1u);
                    umma_commit(t_free);
                    umma_commit(&empty_qe[s]);
                }
                umma_commit(bct);   // also when nothing was issued: the group then stops below
            }
            {
                const bool ok = mbar_wait(bct, pht, wait_ns);
                pht ^= 1u;
                if (group_any(2, kChainThreads, !ok || ut_fail)) { failed = true; break; }
            }
            tc_fence_after();
            if ((warp & 3) >= 2) {   // U -> bf16 (rows in TMEM lanes 64-127)
                const int r = t - 64;
#pragma unroll 1
                for (int jc = 0; jc < NV / 32; ++jc) {
                    float u[32];
                    tmem_ld32(t_UT + lane_q + jc * 32, u);
                    const uint32_t tile = sb + Cfg::OFF_U + ((jc * 32) >> 6) * 8192u;
                    const uint32_t ch0 = ((jc * 32) & 63) >> 3;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const int e = 8 * q4;
                        st_shared_v4(tile + sw128_chunk(r, ch0 + q4), pack_bf16x2(u[e], u[e + 1]),
                                     pack_bf16x2(u[e + 2], u[e + 3]), pack_bf16x2(u[e + 4], u[e + 5]),
                                     pack_bf16x2(u[e + 6], u[e + 7]));
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
            if (t == 0) mbar_arrive(&empty_k[n % 3]);   // MMA_u has read K~ of this stage
            tc_fence_after();
            {
                const int c = t;
                // 2^(G_C - ref) of this chunk, then 2^ref of the next one (unless the
                // next one is handed to the token tail, which takes the plain state).
                // Two multiplies, each rounded, as a call resumed from S_T takes them
                // (S_T, then S0 * 2^ref): resuming is exact to the bit.
                const float gca = gC[(n % 3) * 256 + c];
                const float gcb = (n + 1 < NC && n + 1 < stop_now) ? gC[((n + 1) % 3) * 256 + 128 + c] : 1.f;
                const bool last = (n + 1 == NC);
#pragma unroll 1
                for (int jc = 0; jc < NV / 32; ++jc) {
                    float sv[32];
                    tmem_ld32(t_S + lane_q + jc * 32, sv);
                    if (last && S_T != nullptr && c < DK &&
                        GDN2_IN_BOUNDS(kBufST, S_T + (head * DK + c) * d_v + j0 + jc * 32, 128)) {
                        float4 *dst = reinterpret_cast<float4 *>(S_T + (head * DK + c) * d_v + j0 + jc * 32);
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            dst[e] = make_float4(sv[4 * e] * gca, sv[4 * e + 1] * gca, sv[4 * e + 2] * gca,
                                                 sv[4 * e + 3] * gca);
                    }
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const float2 x = mul_f32x2(mul_f32x2(make_float2(sv[e], sv[e + 1]), make_float2(gca, gca)),
                                                   make_float2(gcb, gcb));
                        sv[e] = x.x;
                        sv[e + 1] = x.y;
                    }
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
                    }
                }
            }
            // fused epilogue: thread t takes the 16-byte column chunk t % (NV / 8) of rows
            // t / (NV / 8) + i * (128 / (NV / 8)); its gate loads are issued here, so that
            // they land while MMA_o runs and o is read out of TMEM
            constexpr int E_CPR = NV / 8, E_RPP = kChainThreads / E_CPR;
            const int e_c16 = t % E_CPR, e_rr = t / E_CPR;
            uint4 gall[EPI ? 64 / E_RPP : 1];
            if constexpr (EPI) {
                const __nv_bfloat16 *gbase = static_cast<const __nv_bfloat16 *>(fz.gate);
#pragma unroll
                for (int i = 0; i < 64 / E_RPP; ++i) {
                    const int r = i * E_RPP + e_rr;
                    const uint4 *gp = reinterpret_cast<const uint4 *>(
                        gbase + ((tok0 + (long)n * 64 + r) * HV + hv) * (long)d_v + j0 + 8 * e_c16);
                    gall[i] = (n * 64 + r < len && GDN2_IN_BOUNDS(kBufGate, gp, 16)) ? __ldg(gp)
                                                                                     : make_uint4(0u, 0u, 0u, 0u);
                }
            }
            {
                const bool ok = mbar_wait(bc3, ph3, wait_ns);
                ph3 ^= 1u;
                if (group_any(2, kChainThreads, !ok)) { failed = true; break; }
            }
            tc_fence_after();
            // O leaves through the U tile (free once MMA_o has run) and one TMA store,
            // except on the partial last chunk of a packed sequence, whose rows past
            // the end belong to the next sequence
            const bool o_tma = !EPI && (!VARLEN || (n + 1) * 64 <= len);
            if ((warp & 3) < (QED ? 1 : 2) && o_tma) {   // QED: the 32 token rows only
                const int r = t;   // output row r (TMEM lanes 0-63)
#pragma unroll 1
                for (int jc = 0; jc < NV / 32; ++jc) {
                    float x[32];
                    tmem_ld32(t_X + lane_q + jc * 32, x);
                    const uint32_t tile = sb + Cfg::OFF_U + ((jc * 32) >> 6) * 8192u;
                    const uint32_t ch0 = ((jc * 32) & 63) >> 3;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const int e = 8 * q4;
                        st_shared_v4(tile + sw128_chunk(r, ch0 + q4), pack_bf16x2(x[e], x[e + 1]),
                                     pack_bf16x2(x[e + 2], x[e + 3]), pack_bf16x2(x[e + 4], x[e + 5]),
                                     pack_bf16x2(x[e + 6], x[e + 7]));
                    }
                }
            } else if ((warp & 3) < 2 && !o_tma) {
                const int r = t;   // output row r (TMEM lanes 0-63); rows past T are padding
                const bool valid = n * 64 + r < len;
                const long orow_off = ((tok0 + (long)n * 64 + r) * HV + hv) * (long)d_v + j0;
                __nv_bfloat16 *orow = o + orow_off;
                bool plain = true;
                if constexpr (EPI) {   // first half of the epilogue: o -> bf16 in the U tile, 1/rms(o) per row
                    plain = false;
                    float ss = 0.f;
#pragma unroll 1
                    for (int jc = 0; jc < NV / 32; ++jc) {
                        float x[32];
                        tmem_ld32(t_X + lane_q + jc * 32, x);
#pragma unroll
                        for (int e = 0; e < 32; ++e) ss = fmaf(x[e], x[e], ss);
                        const uint32_t tile = sb + Cfg::OFF_U + ((jc * 32) >> 6) * 8192u;
                        const uint32_t ch0 = ((jc * 32) & 63) >> 3;
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const int e = 8 * q4;
                            st_shared_v4(tile + sw128_chunk(r, ch0 + q4), pack_bf16x2(x[e], x[e + 1]),
                                         pack_bf16x2(x[e + 2], x[e + 3]), pack_bf16x2(x[e + 4], x[e + 5]),
                                         pack_bf16x2(x[e + 6], x[e + 7]));
                        }
                    }
                    reinterpret_cast<float *>(smem + Cfg::OFF_RMS)[r] = rsqrtf(ss / (float)NV + fz.norm_eps);
                }
#pragma unroll 1
                for (int jc = 0; jc < NV / 32 && plain; ++jc) {
                    float x[32];
                    tmem_ld32(t_X + lane_q + jc * 32, x);
                    if (valid && GDN2_IN_BOUNDS(kBufO, orow + jc * 32, 64)) {
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
            if constexpr (EPI) {   // second half: / rms . weight . silu(g), coalesced, by all four warps
                named_bar(2, kChainThreads);
                const float *nw = reinterpret_cast<const float *>(smem + Cfg::OFF_NW);
                const float *rinv = reinterpret_cast<const float *>(smem + Cfg::OFF_RMS);
                const float4 w0 = *reinterpret_cast<const float4 *>(nw + 8 * e_c16);
                const float4 w1 = *reinterpret_cast<const float4 *>(nw + 8 * e_c16 + 4);
                const float wt[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
                for (int i = 0; i < 64 / E_RPP; ++i) {
                    const int r = i * E_RPP + e_rr;
                    if (n * 64 + r >= len) continue;   // padding rows
                    const long off = ((tok0 + (long)n * 64 + r) * HV + hv) * (long)d_v + j0 + 8 * e_c16;
                    const uint4 gv = gall[i];
                    const float inv = rinv[r];
                    uint32_t a0, a1, a2, a3;
                    ld_shared_v4(sb + Cfg::OFF_U + (e_c16 >> 3) * 8192u + sw128_chunk(r, e_c16 & 7), a0, a1, a2, a3);
                    const uint32_t ov[4] = {a0, a1, a2, a3}, gw[4] = {gv.x, gv.y, gv.z, gv.w};
                    uint32_t pk[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {   // two channels per paired instruction
                        const float2 g2 = make_float2(bf16_lo(gw[e]), bf16_hi(gw[e]));
                        const float2 hx = mul_f32x2(g2, make_float2(0.5f, 0.5f));
                        float2 th;
                        asm("tanh.approx.f32 %0, %1;" : "=f"(th.x) : "f"(hx.x));
                        asm("tanh.approx.f32 %0, %1;" : "=f"(th.y) : "f"(hx.y));
                        const float2 sg = fma_f32x2(th, make_float2(0.5f, 0.5f), make_float2(0.5f, 0.5f));
                        const float2 iw = mul_f32x2(make_float2(inv, inv), make_float2(wt[2 * e], wt[2 * e + 1]));
                        const float2 y = mul_f32x2(mul_f32x2(mul_f32x2(make_float2(bf16_lo(ov[e]), bf16_hi(ov[e])), iw), g2), sg);
                        pk[e] = pack_bf16x2(y.x, y.y);
                    }
                    if (GDN2_IN_BOUNDS(kBufO, o + off, 16))
                        *reinterpret_cast<uint4 *>(o + off) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            }
            tmem_st_wait();
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar(2, kChainThreads);
            if (t == 0) {
                mbar_arrive(&empty_pg[s]);
                if (o_tma) {   // rows past T lie outside the tensor and are not written
#pragma unroll
                    for (int vb = 0; vb < Cfg::VB; ++vb)
                        tma_store_4d(&tm_o, smem + Cfg::OFF_U + vb * 8192, j0 + vb * 64, hv, tma_t0 + n * CH, tma_b);
                    bulk_commit_group();
                }
            }
        }
        if (t == 0) {
            bulk_wait_all();
            umma_commit(&drain[1]);
            mbar_wait(&drain[1], 0u, wait_ns);
        }
    }

    // ------------------------------------------------------------- teardown
    const bool any_failed = __syncthreads_or(failed);
    if (any_failed && tid == 0) record_timeout();
    // every role has stopped at the same chunk and drained its loads, MMAs and stores
    const int len_s = reinterpret_cast<const int *>(smem + Cfg::OFF_SEQ)[2];
    const int nc_s = (len_s + CH - 1) / CH;
    const int stop = any_failed ? nc_s : min(nc_s, *stop_at);
    if (stop < nc_s && warp >= 8 && warp < 12) {   // the chain warps copy the state out of TMEM
        tc_fence_after();
        float *sS = reinterpret_cast<float *>(smem);
        const int c = tid - kKeyThreads;
#pragma unroll 1
        for (int jc = 0; jc < NV / 32; ++jc) {
            float x[32];
            tmem_ld32(t_S + lane_q + jc * 32, x);
            if (c < DK) {
#pragma unroll
                for (int e = 0; e < 32; e += 4)
                    *reinterpret_cast<float4 *>(sS + c * (NV + 4) + jc * 32 + e) =
                        make_float4(x[e], x[e + 1], x[e + 2], x[e + 3]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, Cfg::TMEM_COLS);
    }
    if (stop < nc_s) {
        const long tok0_s = *reinterpret_cast<const long *>(smem + Cfg::OFF_SEQ);
        const int bb_s = reinterpret_cast<const int *>(smem + Cfg::OFF_SEQ)[3];
        const int hv_s = blockIdx.y;
        if constexpr (QED)
            tc_token_tail_qed<DK, NV>(smem, ta, la, o, S_T, tok0_s, stop * CH, len_s, hv_s, H, blockIdx.x * NV, d_v,
                                      (long)bb_s * HV + hv_s);
        else
            tc_token_tail<DK, NV, PREP, EPI>(smem, ta, la, o, S_T, tok0_s, stop * CH, len_s, hv_s / (HV / H), H,
                                             hv_s, HV, blockIdx.x * NV, d_v, (long)bb_s * HV + hv_s, fz);
    }
}

}  // namespace gdn2
