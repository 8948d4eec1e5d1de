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
// Layout: one block of 256 threads per (head, 64- or 128-column slice of
// d_v).  A row of the slice is NVD floats: NVD/4 threads each own a float4
// column group, the remaining thread rows each own DK / (256 / (NVD/4)) rows.
// Every thread issues all its 128-bit loads of S before any arithmetic, so a
// block keeps 32-64 KB of HBM reads in flight.  Column sums over d_k are
// reduced through shared memory.
#pragma once
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

template <typename IO, int DK, int NVD>
__global__ void __launch_bounds__(256, 2)
decode_step_kernel(const IO *__restrict__ q, const IO *__restrict__ k, const IO *__restrict__ v,
                   const IO *__restrict__ la, const IO *__restrict__ bg, const IO *__restrict__ wg,
                   float *__restrict__ S, IO *__restrict__ o, int d_v) {
    constexpr int TPR = NVD / 4;   // threads across one row of the slice
    constexpr int RG = 256 / TPR;  // thread rows
    constexpr int RPT = DK / RG;   // state rows per thread
    static_assert(RPT >= 1 && RG * RPT == DK, "bad decode tiling");

    __shared__ float s_alpha[DK], s_erase[DK], s_qa[DK], s_k[DK];
    __shared__ float s_wv[NVD];
    __shared__ __align__(16) float s_red_r[RG][NVD];
    __shared__ __align__(16) float s_red_p[RG][NVD];
    __shared__ float s_qk[8];

    const int tid = threadIdx.x;
    const int cg = tid % TPR;        // float4 column group
    const int rg = tid / TPR;        // thread row
    const long bh = blockIdx.x;      // flat b * H + h
    const int j0 = blockIdx.y * NVD;

    float *Sh = S + bh * (long)DK * d_v + j0 + cg * 4;
    float4 s[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int row = i * RG + rg;
        s[i] = __ldcs(reinterpret_cast<const float4 *>(Sh + (long)row * d_v));
    }

    // per-row and per-column coefficients
    const IO *qh = q + bh * DK, *kh = k + bh * DK, *lah = la + bh * DK, *bh_ = bg + bh * DK;
    float qk = 0.f;
    if (tid < DK) {
        const float a = __expf(ld_io(lah + tid));
        const float kv = ld_io(kh + tid);
        const float qv = ld_io(qh + tid);
        s_alpha[tid] = a;
        s_erase[tid] = ld_io(bh_ + tid) * kv * a;
        s_qa[tid] = qv * a;
        s_k[tid] = kv;
        qk = qv * kv;
    }
    if (tid < NVD) {
        const long vo = bh * (long)d_v + j0 + tid;
        s_wv[tid] = ld_io(wg + vo) * ld_io(v + vo);
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

    if (rg == 0) {
#pragma unroll
        for (int g = 0; g < RG; ++g) {
            const float4 a = *reinterpret_cast<const float4 *>(&s_red_p[g][cg * 4]);
            pt.x += a.x; pt.y += a.y; pt.z += a.z; pt.w += a.w;
        }
        float qkt = 0.f;
#pragma unroll
        for (int wi = 0; wi < (DK + 31) / 32; ++wi) qkt += s_qk[wi];
        st_io4<IO>(o + bh * (long)d_v + j0 + cg * 4, pt.x + qkt * u.x, pt.y + qkt * u.y, pt.z + qkt * u.z,
                   pt.w + qkt * u.w);
    }

#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int row = i * RG + rg;
        const float a = s_alpha[row], kv = s_k[row];
        float4 n;
        n.x = a * s[i].x + kv * u.x;
        n.y = a * s[i].y + kv * u.y;
        n.z = a * s[i].z + kv * u.z;
        n.w = a * s[i].w + kv * u.w;
        __stcs(reinterpret_cast<float4 *>(Sh + (long)row * d_v), n);
    }
}

}  // namespace gdn2
