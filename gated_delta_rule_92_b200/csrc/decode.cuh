// decode.cuh -- fused single-token decode step of the GDN-2 recurrence.
//
// burn-gdn2 README, "Architecture": S_t = (I - k (b.k)^T) diag(alpha) S_{t-1}
// + k (w.v)^T and o_t = S_t^T q; the README's "Fused Recurrent (infer)" mode
// carries S between calls.  Per (b, h) and value column j, with S = S_{t-1}:
//     r_j = sum_i (b_i k_i alpha_i) S_ij        erase read-out   (k^T S after decay)
//     p_j = sum_i (q_i alpha_i) S_ij            q^T of the decayed state
//     u_j = w_j v_j - r_j
//     S_ij <- alpha_i S_ij + k_i u_j
//     o_j  = p_j + (q . k) u_j                  = q^T S_t
// so S is read once and written once; everything else is a few KB.
//
// Layout: one block of 256 threads per (value head, 64- or 128-column slice
// of d_v); with HV = G H value heads (num_v_heads), value head hv reads key
// head hv / G.  A row of the slice is NVD floats: NVD/4 threads each own a float4
// column group, the remaining thread rows each own DK / (256 / (NVD/4)) rows.
// Every thread issues all its 128-bit loads of S before any arithmetic, so a
// block keeps 32-64 KB of HBM reads in flight.  Column sums over d_k are
// reduced through shared memory.
#pragma once
#include <cooperative_groups.h>

#include "gdn2_device.cuh"

namespace gdn2 {

template <typename T>
__device__ __forceinline__ float ld_io(const T *p);
template <>
__device__ __forceinline__ float ld_io<float>(const float *p) { return __ldg(p); }
template <>
__device__ __forceinline__ float ld_io<__nv_bfloat16>(const __nv_bfloat16 *p) {
    return __bfloat162float(__ldg(p));
}

template <typename IO>
__device__ __forceinline__ void st_io4(IO *p, float a, float b, float c, float d);
template <>
__device__ __forceinline__ void st_io4<float>(float *p, float a, float b, float c, float d) {
    *reinterpret_cast<float4 *>(p) = make_float4(a, b, c, d);
}
template <>
__device__ __forceinline__ void st_io4<__nv_bfloat16>(__nv_bfloat16 *p, float a, float b, float c, float d) {
    uint2 u;
    u.x = pack_bf16x2(a, b);
    u.y = pack_bf16x2(c, d);
    *reinterpret_cast<uint2 *>(p) = u;
}

// Optional fusion around the step (burn-gdn2 README, "Architecture": the
// L2-Norm before the mixer and the SiLU-gated RMS norm after it;
// "Configuration": allow_neg_eigval, norm_eps).
struct FuseArgs {
    int prep;                  // q, k, b, w raw: L2-normalise q, k; b, w = sigmoid
    int neg_eigval;            // with prep: b = 2 sigmoid(b_raw)
    float l2_eps;
    const void *gate;          // non-null: y = o / sqrt(mean(o^2) + eps) * weight * silu(gate)
    const float *norm_weight;  // [d_v]
    float norm_eps;
};

template <typename IO>
__device__ __forceinline__ float sigmoid_io(float x) {
    if constexpr (sizeof(IO) == 4) return sigmoid_f32(x);
    else return sigmoid_tanh(x);
}

// With FUSED, the d_v / NVD blocks of one (b, h) form a thread-block cluster
// along y when the epilogue is on and d_v > NVD, so the RMS over d_v can add
// the blocks' partial sums through distributed shared memory.
template <typename IO, int DK, int NVD, bool FUSED = false>
__global__ void __launch_bounds__(256, 2)
decode_step_kernel(const IO *__restrict__ q, const IO *__restrict__ k, const IO *__restrict__ v,
                   const IO *__restrict__ la, const IO *__restrict__ bg, const IO *__restrict__ wg,
                   float *__restrict__ S, IO *__restrict__ o, int d_v, int H, int HV, FuseArgs fz = {}) {
    constexpr int TPR = NVD / 4;   // threads across one row of the slice
    constexpr int RG = 256 / TPR;  // thread rows
    constexpr int RPT = DK / RG;   // state rows per thread
    static_assert(RPT >= 1 && RG * RPT == DK, "bad decode tiling");

    __shared__ float s_alpha[DK], s_erase[DK], s_qa[DK], s_k[DK];
    __shared__ float s_wv[NVD];
    __shared__ __align__(16) float s_red_r[RG][NVD];
    __shared__ __align__(16) float s_red_p[RG][NVD];
    __shared__ float s_qk[8];
    __shared__ float s_nrm[2][8];      // fused prep: per-warp sums of q^2, k^2
    __shared__ float s_ss[8];          // fused epilogue: sum of o^2 per block of the cluster

    const int tid = threadIdx.x;
    const int cg = tid % TPR;        // float4 column group
    const int rg = tid / TPR;        // thread row
    const int bhi = blockIdx.x;      // flat b * HV + hv (value head; state, v, w, o); B HV <= INT_MAX
    const long bh = bhi;
    // its key head (q, k, log_alpha, b)
    const long bk = (HV == H) ? bh : (long)((bhi / HV) * H + (bhi % HV) / (HV / H));
    const int j0 = blockIdx.y * NVD;

    float *Sh = S + bh * (long)DK * d_v + j0 + cg * 4;
    float4 s[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int row = i * RG + rg;
        const float4 *sp = reinterpret_cast<const float4 *>(Sh + (long)row * d_v);
        s[i] = GDN2_IN_BOUNDS(kBufS0, sp, 16) ? __ldcs(sp) : make_float4(0.f, 0.f, 0.f, 0.f);
    }

    // fused epilogue: its gate and weight values are read now, under the state loads
    float gate4[4] = {0.f, 0.f, 0.f, 0.f};
    float4 wt4 = make_float4(0.f, 0.f, 0.f, 0.f);
    if constexpr (FUSED) {
        if (fz.gate != nullptr && rg == 0) {
            const IO *gp = static_cast<const IO *>(fz.gate) + bh * (long)d_v + j0 + cg * 4;
#pragma unroll
            for (int e = 0; e < 4; ++e) gate4[e] = GDN2_IN_BOUNDS(kBufGate, gp + e, sizeof(IO)) ? ld_io(gp + e) : 0.f;
            const float4 *wp = reinterpret_cast<const float4 *>(fz.norm_weight + j0 + cg * 4);
            if (GDN2_IN_BOUNDS(kBufNW, wp, 16)) wt4 = __ldg(wp);
        }
    }

    // per-row and per-column coefficients
    const IO *qh = q + bk * DK, *kh = k + bk * DK, *lah = la + bk * DK, *bh_ = bg + bk * DK;
    float qk = 0.f;
    float kv = 0.f, qv = 0.f, bv = 0.f;
    if (tid < DK) {
        kv = GDN2_IN_BOUNDS(kBufK, kh + tid, sizeof(IO)) ? ld_io(kh + tid) : 0.f;
        qv = GDN2_IN_BOUNDS(kBufQ, qh + tid, sizeof(IO)) ? ld_io(qh + tid) : 0.f;
        bv = GDN2_IN_BOUNDS(kBufB, bh_ + tid, sizeof(IO)) ? ld_io(bh_ + tid) : 0.f;
    }
    if constexpr (FUSED) {
        if (fz.prep) {   // q / |q|, k / |k| over d_k (block reduction), sigmoid gates
            float sq = qv * qv, sk = kv * kv;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                sq += __shfl_xor_sync(0xffffffffu, sq, off);
                sk += __shfl_xor_sync(0xffffffffu, sk, off);
            }
            if ((tid & 31) == 0 && tid < DK) { s_nrm[0][tid >> 5] = sq; s_nrm[1][tid >> 5] = sk; }
            __syncthreads();
            sq = 0.f;
            sk = 0.f;
#pragma unroll
            for (int wi = 0; wi < DK / 32; ++wi) { sq += s_nrm[0][wi]; sk += s_nrm[1][wi]; }
            qv *= l2_inv(sq, fz.l2_eps);
            kv *= l2_inv(sk, fz.l2_eps);
            bv = (fz.neg_eigval ? 2.f : 1.f) * sigmoid_io<IO>(bv);
        }
    }
    if (tid < DK) {
        const float a = __expf(GDN2_IN_BOUNDS(kBufLA, lah + tid, sizeof(IO)) ? ld_io(lah + tid) : 0.f);
        s_alpha[tid] = a;
        s_erase[tid] = bv * kv * a;
        s_qa[tid] = qv * a;
        s_k[tid] = kv;
        qk = qv * kv;
    }
    if (tid < NVD) {
        const long vo = bh * (long)d_v + j0 + tid;
        float wv = GDN2_IN_BOUNDS(kBufW, wg + vo, sizeof(IO)) ? ld_io(wg + vo) : 0.f;
        if constexpr (FUSED) {
            if (fz.prep) wv = sigmoid_io<IO>(wv);
        }
        s_wv[tid] = wv * (GDN2_IN_BOUNDS(kBufV, v + vo, sizeof(IO)) ? ld_io(v + vo) : 0.f);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) qk += __shfl_xor_sync(0xffffffffu, qk, off);
    if ((tid & 31) == 0) s_qk[tid >> 5] = qk;
    __syncthreads();

    // partial column sums over this thread's rows
    float4 r4 = make_float4(0.f, 0.f, 0.f, 0.f), p4 = r4;
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int row = i * RG + rg;
        const float e = s_erase[row], qa = s_qa[row];
        r4.x += e * s[i].x; r4.y += e * s[i].y; r4.z += e * s[i].z; r4.w += e * s[i].w;
        p4.x += qa * s[i].x; p4.y += qa * s[i].y; p4.z += qa * s[i].z; p4.w += qa * s[i].w;
    }
    *reinterpret_cast<float4 *>(&s_red_r[rg][cg * 4]) = r4;
    *reinterpret_cast<float4 *>(&s_red_p[rg][cg * 4]) = p4;
    __syncthreads();

    float4 rt = make_float4(0.f, 0.f, 0.f, 0.f), pt = rt;
#pragma unroll
    for (int g = 0; g < RG; ++g) {
        const float4 a = *reinterpret_cast<const float4 *>(&s_red_r[g][cg * 4]);
        rt.x += a.x; rt.y += a.y; rt.z += a.z; rt.w += a.w;
    }
    const float4 wv = *reinterpret_cast<const float4 *>(&s_wv[cg * 4]);
    const float4 u = make_float4(wv.x - rt.x, wv.y - rt.y, wv.z - rt.z, wv.w - rt.w);

    float4 ov = make_float4(0.f, 0.f, 0.f, 0.f);
    if (rg == 0) {
#pragma unroll
        for (int g = 0; g < RG; ++g) {
            const float4 a = *reinterpret_cast<const float4 *>(&s_red_p[g][cg * 4]);
            pt.x += a.x; pt.y += a.y; pt.z += a.z; pt.w += a.w;
        }
        float qkt = 0.f;
#pragma unroll
        for (int wi = 0; wi < (DK + 31) / 32; ++wi) qkt += s_qk[wi];
        ov = make_float4(pt.x + qkt * u.x, pt.y + qkt * u.y, pt.z + qkt * u.z, pt.w + qkt * u.w);
    }
    // the state update goes out before the epilogue's synchronisation
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int row = i * RG + rg;
        const float a = s_alpha[row], kv = s_k[row];
        float4 n;
        n.x = a * s[i].x + kv * u.x;
        n.y = a * s[i].y + kv * u.y;
        n.z = a * s[i].z + kv * u.z;
        n.w = a * s[i].w + kv * u.w;
        float4 *sp = reinterpret_cast<float4 *>(Sh + (long)row * d_v);
        if (GDN2_IN_BOUNDS(kBufST, sp, 16)) __stcs(sp, n);
    }

    bool plain_store = true;
    if constexpr (FUSED) {
        if (fz.gate != nullptr) {   // gated RMS norm over the whole d_v row
            plain_store = false;
            float ss = ov.x * ov.x + ov.y * ov.y + ov.z * ov.z + ov.w * ov.w;   // zero for rg != 0
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
            const int nblk = d_v / NVD;   // cluster size along y (1: no cluster)
            if (nblk == 1) {
                if (tid == 0) s_ss[0] = ss;
                __syncthreads();
            } else {
                // every block of the cluster has started before any writes into a
                // peer's shared memory; the second sync publishes the sums
                cooperative_groups::cluster_group cl = cooperative_groups::this_cluster();
                cl.sync();
                if (tid == 0)
                    for (int r = 0; r < nblk; ++r) cl.map_shared_rank(s_ss, r)[blockIdx.y] = ss;
                cl.sync();
            }
            if (rg == 0) {
                float tot = 0.f;
                for (int r = 0; r < nblk; ++r) tot += s_ss[r];
                const float inv = rsqrtf(tot / (float)d_v + fz.norm_eps);
                const long go = bh * (long)d_v + j0 + cg * 4;
                const float4 wt = wt4;
                const float g0 = gate4[0], g1 = gate4[1], g2 = gate4[2], g3 = gate4[3];
                if (GDN2_IN_BOUNDS(kBufO, o + go, 4 * sizeof(IO)))
                    st_io4<IO>(o + go, ov.x * inv * wt.x * g0 * sigmoid_io<IO>(g0),
                               ov.y * inv * wt.y * g1 * sigmoid_io<IO>(g1),
                               ov.z * inv * wt.z * g2 * sigmoid_io<IO>(g2),
                               ov.w * inv * wt.w * g3 * sigmoid_io<IO>(g3));
            }
        }
    }
    if (plain_store && rg == 0 && GDN2_IN_BOUNDS(kBufO, o + bh * (long)d_v + j0 + cg * 4, 4 * sizeof(IO)))
        st_io4<IO>(o + bh * (long)d_v + j0 + cg * 4, ov.x, ov.y, ov.z, ov.w);
}

}  // namespace gdn2
