// epilogue.cuh -- the gated RMS norm after the mixer, as its own pass.
//
// burn-gdn2 README, "Architecture" (Gated RMS Norm <- SiLU Gate) and
// "Configuration" (norm_eps): per (token, head) row of d_v,
//     y_j = o_j / sqrt(mean_j o_j^2 + eps) * weight_j * silu(g_j),
//     silu(x) = x sigmoid(x).
// The chunk kernels apply this while o is still in registers whenever one CTA
// holds the whole row; this kernel covers the other cases (d_v split across
// CTAs), in place over o.  One warp per row.
#pragma once
#include "decode.cuh"

namespace gdn2 {

template <typename IO>
__global__ void __launch_bounds__(256)
gated_rmsnorm_kernel(IO *__restrict__ o, const IO *__restrict__ g, const float *__restrict__ weight, long rows,
                     int d_v, float eps) {
    const long row = (long)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int l = threadIdx.x & 31;
    IO *orow = o + row * d_v;
    const IO *grow = g + row * d_v;
    float ss = 0.f;
    for (int j = l; j < d_v; j += 32) {
        const float x = GDN2_IN_BOUNDS(kBufO, orow + j, sizeof(IO)) ? ld_io(orow + j) : 0.f;
        ss = fmaf(x, x, ss);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float inv = rsqrtf(ss / (float)d_v + eps);
    for (int j = l; j < d_v; j += 32) {
        if (!GDN2_IN_BOUNDS(kBufO, orow + j, sizeof(IO)) || !GDN2_IN_BOUNDS(kBufGate, grow + j, sizeof(IO)) ||
            !GDN2_IN_BOUNDS(kBufNW, weight + j, sizeof(float)))
            continue;
        const float x = ld_io(orow + j), gv = ld_io(grow + j);
        const float y = x * inv * __ldg(weight + j) * gv * sigmoid_io<IO>(gv);
        if constexpr (sizeof(IO) == 4) orow[j] = y;
        else orow[j] = __float2bfloat16_rn(y);
    }
}

}  // namespace gdn2
