// gdn2_lib.cu -- the C ABI declared in include/gdn2.h.
//
// One translation unit: it includes every kernel header, validates
// arguments on the host, encodes the TMA tensor maps and launches on the
// caller's stream.  Nothing here allocates device memory.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <climits>
#include <cstring>
#include <atomic>
#include <mutex>

#include "../../include/gdn2.h"
#include "chunk_ffma.cuh"
#include "chunk_tc.cuh"
#include "decode.cuh"
#include "epilogue.cuh"
#include "qed.cuh"
#include "gdn2_device.cuh"

namespace gdn2 {

// Default bound on any single device-side wait (2 s): far above any wait a
// correct launch performs, short enough that a stuck kernel returns.
constexpr unsigned long long kWaitNs = 2000000000ull;

__global__ void selftest_wait_kernel(unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        // Nothing arrives on this barrier, so phase 0 never completes.
        if (!mbar_wait(&bar, 0u, limit_ns)) record_timeout();
    }
}

#ifdef GDN2_DEBUG_BOUNDS
// Debug build: publishes one call's buffer extents, in stream order (a kernel
// parameter, so the write can also be captured into a CUDA graph).
__global__ void set_bounds_kernel(BoundsTable t) { g_bounds = t; }

// Exercises the range check on addresses only (nothing is dereferenced): an
// 8-byte range inside a 64-byte extent passes, one that runs past its end
// fails and records GDN2_ERR_OUT_OF_BOUNDS with this buffer and line.  A check
// that answers wrongly leaves GDN2_ERR_INVALID_ARG instead.
__global__ void selftest_bounds_kernel(unsigned long long fake_base) {
    g_bounds.lo[kBufQ] = fake_base;
    g_bounds.hi[kBufQ] = fake_base + 64;
    const char *base = reinterpret_cast<const char *>(fake_base);
    const bool inside = GDN2_IN_BOUNDS(kBufQ, base + 56, 8);
    const bool past_end = GDN2_IN_BOUNDS(kBufQ, base + 60, 8);
    if (!inside || past_end) record_status(kStatusBadArgs);
}
#endif

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

gdn2_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? GDN2_OK : GDN2_ERR_CUDA; }

// Injected launch failures (gdn2_testing_fail_launches): after `pass` more
// launches, the next `fail` launch sites return GDN2_ERR_CUDA without
// launching, as a failed launch would.  Disarmed (the default) it costs one
// relaxed atomic load per launch.
std::atomic<bool> g_inject_armed{false};
std::mutex g_inject_lock;
long g_inject_pass = 0, g_inject_fail = 0;

gdn2_status_t launch_gate() {
    if (!g_inject_armed.load(std::memory_order_relaxed)) return GDN2_OK;
    std::lock_guard<std::mutex> guard(g_inject_lock);
    if (g_inject_fail <= 0) return GDN2_OK;
    if (g_inject_pass > 0) {
        --g_inject_pass;
        return GDN2_OK;
    }
    if (--g_inject_fail == 0) g_inject_armed.store(false, std::memory_order_relaxed);
    return GDN2_ERR_CUDA;
}

// The extents of one call's buffers for the debug build's device-side range
// checks (bounds.cuh), from the call's pointers and the layouts of gdn2.h;
// the release build does nothing here.  `e` is the bytes of one token element.
struct CallBounds {
    BoundsTable t{};
    void add(int buf, const void *p, size_t bytes) {
        if (p == nullptr) return;
        t.lo[buf] = reinterpret_cast<uintptr_t>(p);
        t.hi[buf] = t.lo[buf] + bytes;
    }
    gdn2_status_t publish(cudaStream_t st) const {
#ifdef GDN2_DEBUG_BOUNDS
        set_bounds_kernel<<<1, 1, 0, st>>>(t);
        return from_cuda(cudaGetLastError());
#else
        (void)st;
        return GDN2_OK;
#endif
    }
};

#ifdef GDN2_DEBUG_BOUNDS
constexpr bool kDebugBounds = true;
#else
constexpr bool kDebugBounds = false;
#endif

// token tensors [B', T, H | HV, d] (B' = 1 with cu_seqlens), states [B, HV, d_k, d_v]
gdn2_status_t bounds_chunk(const void *q, const void *k, const void *v, const void *la, const void *b,
                           const void *c, const void *w, const float *S0, const void *o, const float *S_T, int B,
                           int Bt, int T, int H, int HV, int d_k, int d_v, const int *cu, size_t e,
                           const FuseArgs *fz, cudaStream_t st) {
    if (!kDebugBounds) return GDN2_OK;
    CallBounds cb;
    const size_t ntok = (size_t)Bt * T;
    const size_t kb = ntok * H * d_k * e, vb = ntok * HV * d_v * e;
    const size_t sb = (size_t)B * HV * d_k * d_v * sizeof(float);
    cb.add(kBufQ, q, kb);
    cb.add(kBufK, k, kb);
    cb.add(kBufLA, la, kb);
    cb.add(kBufB, b, kb);
    cb.add(kBufC, c, kb);
    cb.add(kBufV, v, vb);
    cb.add(kBufW, w, vb);
    cb.add(kBufO, o, vb);
    cb.add(kBufS0, S0, sb);
    cb.add(kBufST, S_T, sb);
    if (fz != nullptr && fz->gate != nullptr) {
        cb.add(kBufGate, fz->gate, vb);
        cb.add(kBufNW, fz->norm_weight, (size_t)d_v * sizeof(float));
    }
    cb.add(kBufCU, cu, (size_t)(B + 1) * sizeof(int));
    return cb.publish(st);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// Token tensor [B, T, H, d] bf16 viewed as 4-D (d, H, T, B); box = 64 channels
// x 1 head x `rows` tokens (64, or 32 for the QED chunks) x 1 sequence,
// 128-byte swizzle.  Boxes that run past T are zero-filled by the TMA unit (a
// partial last chunk).
bool make_token_map(CUtensorMap *m, const void *base, int B, int T, int H, int d, int rows = 64) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)d * 2u, (cuuint64_t)H * (cuuint64_t)d * 2u,
                             (cuuint64_t)T * (cuuint64_t)H * (cuuint64_t)d * 2u};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)rows, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Problem shape shared by the launchers: B sequences of T tokens, or, with
// cu_seqlens, B sequences packed along T tokens; H key heads, HV value heads.
struct Shape {
    int B, T, H, HV, d_k, d_v;
    const int *cu;      // device [B + 1] or null
    int tensor_b() const { return cu ? 1 : B; }   // leading dim of the token tensors
    long rows() const { return (long)tensor_b() * T * HV; }   // (token, value head) rows of o
};

template <typename IO>
gdn2_status_t launch_rmsnorm(void *o, const void *g, const float *weight, long rows, int d_v, float eps,
                             cudaStream_t st) {
    if (rows == 0) return GDN2_OK;
    if (launch_gate() != GDN2_OK) return GDN2_ERR_CUDA;
    gated_rmsnorm_kernel<IO><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(
        static_cast<IO *>(o), static_cast<const IO *>(g), weight, rows, d_v, eps);
    return from_cuda(cudaGetLastError());
}

template <int DK, int NV, bool PREP, bool EPI, bool VARLEN>
gdn2_status_t launch_tc_kernel(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tb,
                               const CUtensorMap &tv, const CUtensorMap &tw, const CUtensorMap &to, const void *la,
                               const float *S0,
                               void *o, float *S_T, const Shape &sh, cudaStream_t st, const FuseArgs &fz,
                               const TailArgs &ta) {
    if (launch_gate() != GDN2_OK) return GDN2_ERR_CUDA;
    using Cfg = TcCfg<DK, NV>;
    auto kern = chunk_fwd_tc_kernel<DK, NV, PREP, EPI, VARLEN>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::SMEM_ALLOC);
    if (e != cudaSuccess) return GDN2_ERR_CUDA;
    dim3 grid(sh.d_v / NV, sh.HV, sh.B);
    kern<<<grid, kTcThreads, Cfg::SMEM_ALLOC, st>>>(tq, tk, tb, tv, tw, to, tq, static_cast<const __nv_bfloat16 *>(la),
                                                    S0, static_cast<__nv_bfloat16 *>(o), S_T, sh.T, sh.H, sh.HV,
                                                    sh.d_v, sh.cu, kWaitNs, fz, ta);
    return from_cuda(cudaGetLastError());
}

// Packed sequences take the kernel built with the per-sequence offsets; the
// equal-length one has none of that code.
template <int DK, int NV, bool PREP, bool EPI>
gdn2_status_t launch_tc_seq(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tb,
                            const CUtensorMap &tv, const CUtensorMap &tw, const CUtensorMap &to, const void *la,
                            const float *S0, void *o, float *S_T, const Shape &sh, cudaStream_t st,
                            const FuseArgs &fz, const TailArgs &ta) {
    if (sh.cu)
        return launch_tc_kernel<DK, NV, PREP, EPI, true>(tq, tk, tb, tv, tw, to, la, S0, o, S_T, sh, st, fz, ta);
    return launch_tc_kernel<DK, NV, PREP, EPI, false>(tq, tk, tb, tv, tw, to, la, S0, o, S_T, sh, st, fz, ta);
}

template <int DK, int NV>
gdn2_status_t launch_tc(const void *q, const void *k, const void *v, const void *la, const void *b, const void *w,
                        const float *S0, void *o, float *S_T, const Shape &sh, cudaStream_t st,
                        const FuseArgs *fz = nullptr) {
    CUtensorMap tq, tk, tb, tv, tw, to;
    const int Bt = sh.tensor_b();
    if (!make_token_map(&tq, q, Bt, sh.T, sh.H, DK) || !make_token_map(&tk, k, Bt, sh.T, sh.H, DK) ||
        !make_token_map(&tb, b, Bt, sh.T, sh.H, DK) || !make_token_map(&tv, v, Bt, sh.T, sh.HV, sh.d_v) ||
        !make_token_map(&tw, w, Bt, sh.T, sh.HV, sh.d_v) || !make_token_map(&to, o, Bt, sh.T, sh.HV, sh.d_v))
        return GDN2_ERR_CUDA;
    const bool prep = fz != nullptr && fz->prep;
    // the in-kernel epilogue needs the whole d_v row in one CTA; otherwise one
    // more pass normalises o in place
    const bool epi = fz != nullptr && fz->gate != nullptr && sh.d_v == NV;
    const FuseArgs kf = fz ? *fz : FuseArgs{};
    const TailArgs ta{static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k),
                      static_cast<const __nv_bfloat16 *>(b), static_cast<const __nv_bfloat16 *>(v),
                      static_cast<const __nv_bfloat16 *>(w)};
    gdn2_status_t s;
    if (prep && epi) s = launch_tc_seq<DK, NV, true, true>(tq, tk, tb, tv, tw, to, la, S0, o, S_T, sh, st, kf, ta);
    else if (prep) s = launch_tc_seq<DK, NV, true, false>(tq, tk, tb, tv, tw, to, la, S0, o, S_T, sh, st, kf, ta);
    else if (epi) s = launch_tc_seq<DK, NV, false, true>(tq, tk, tb, tv, tw, to, la, S0, o, S_T, sh, st, kf, ta);
    else s = launch_tc_seq<DK, NV, false, false>(tq, tk, tb, tv, tw, to, la, S0, o, S_T, sh, st, kf, ta);
    if (s != GDN2_OK || fz == nullptr || fz->gate == nullptr || epi) return s;
    return launch_rmsnorm<__nv_bfloat16>(o, fz->gate, fz->norm_weight, sh.rows(), sh.d_v, fz->norm_eps, st);
}

// The second erase direction on the tensor-core kernel (bf16 I/O): 32 tokens a
// chunk, token maps with 32-row boxes, the gate c through its own map.
template <int DK, int NV>
gdn2_status_t launch_tc_qed(const void *q, const void *k, const void *v, const void *la, const void *b,
                            const void *c, const void *w, const float *S0, void *o, float *S_T, int B, int T, int H,
                            int d_v, float eps, cudaStream_t st) {
    if (launch_gate() != GDN2_OK) return GDN2_ERR_CUDA;
    using Cfg = TcCfg<DK, NV>;
    CUtensorMap tq, tk, tb, tc, tv, tw, to;
    if (!make_token_map(&tq, q, B, T, H, DK, 32) || !make_token_map(&tk, k, B, T, H, DK, 32) ||
        !make_token_map(&tb, b, B, T, H, DK, 32) || !make_token_map(&tc, c, B, T, H, DK, 32) ||
        !make_token_map(&tv, v, B, T, H, d_v, 32) || !make_token_map(&tw, w, B, T, H, d_v, 32) ||
        !make_token_map(&to, o, B, T, H, d_v, 32))
        return GDN2_ERR_CUDA;
    auto kern = chunk_fwd_tc_kernel<DK, NV, false, false, false, true>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::SMEM_ALLOC) != cudaSuccess)
        return GDN2_ERR_CUDA;
    TailArgs ta{static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k),
                static_cast<const __nv_bfloat16 *>(b), static_cast<const __nv_bfloat16 *>(v),
                static_cast<const __nv_bfloat16 *>(w)};
    ta.c = static_cast<const __nv_bfloat16 *>(c);
    ta.qed_eps = eps;
    dim3 grid(d_v / NV, H, B);
    kern<<<grid, kTcThreads, Cfg::SMEM_ALLOC, st>>>(tq, tk, tb, tv, tw, to, tc, static_cast<const __nv_bfloat16 *>(la),
                                                    S0, static_cast<__nv_bfloat16 *>(o), S_T, T, H, H, d_v, nullptr,
                                                    kWaitNs, FuseArgs{}, ta);
    return from_cuda(cudaGetLastError());
}

template <typename IO, int DK, int CH>
gdn2_status_t launch_ffma(const void *q, const void *k, const void *v, const void *la, const void *b,
                          const void *w, const float *S0, void *o, float *S_T, const Shape &sh, cudaStream_t st,
                          const FuseArgs *fz = nullptr) {
    if (launch_gate() != GDN2_OK) return GDN2_ERR_CUDA;
    using Cfg = FfmaCfg<DK, CH>;
    dim3 grid(sh.d_v / Cfg::NV, sh.HV, sh.B);
    const IO *qp = static_cast<const IO *>(q), *kp = static_cast<const IO *>(k), *vp = static_cast<const IO *>(v);
    const IO *lp = static_cast<const IO *>(la), *bp = static_cast<const IO *>(b), *wp = static_cast<const IO *>(w);
    IO *op = static_cast<IO *>(o);
    if (fz == nullptr) {
        auto kern = chunk_fwd_ffma_kernel<IO, DK, false, CH>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::BYTES);
        if (e != cudaSuccess) return GDN2_ERR_CUDA;
        kern<<<grid, 256, Cfg::BYTES, st>>>(qp, kp, vp, lp, bp, wp, S0, op, S_T, sh.T, sh.H, sh.HV, sh.d_v, sh.cu,
                                            FuseArgs{});
        return from_cuda(cudaGetLastError());
    }
    auto kern = chunk_fwd_ffma_kernel<IO, DK, true, CH>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::BYTES);
    if (e != cudaSuccess) return GDN2_ERR_CUDA;
    kern<<<grid, 256, Cfg::BYTES, st>>>(qp, kp, vp, lp, bp, wp, S0, op, S_T, sh.T, sh.H, sh.HV, sh.d_v, sh.cu, *fz);
    gdn2_status_t s = from_cuda(cudaGetLastError());
    if (s != GDN2_OK || fz->gate == nullptr) return s;
    return launch_rmsnorm<IO>(o, fz->gate, fz->norm_weight, sh.rows(), sh.d_v, fz->norm_eps, st);
}

template <typename IO, int DK, int NVD>
gdn2_status_t launch_decode(const void *q, const void *k, const void *v, const void *la, const void *b,
                            const void *w, float *S, void *o, int B, int H, int HV, int d_v, cudaStream_t st,
                            const FuseArgs *fz) {
    if (launch_gate() != GDN2_OK) return GDN2_ERR_CUDA;
    // the state is read and written in place: both extents are S
    gdn2_status_t s = bounds_chunk(q, k, v, la, b, nullptr, w, S, o, S, B, B, 1, H, HV, DK, d_v, nullptr, sizeof(IO),
                                   fz, st);
    if (s != GDN2_OK) return s;
    dim3 grid((unsigned)((long)B * HV), d_v / NVD);
    if (fz == nullptr) {
        decode_step_kernel<IO, DK, NVD><<<grid, 256, 0, st>>>(
            static_cast<const IO *>(q), static_cast<const IO *>(k), static_cast<const IO *>(v),
            static_cast<const IO *>(la), static_cast<const IO *>(b), static_cast<const IO *>(w), S,
            static_cast<IO *>(o), d_v, H, HV, FuseArgs{});
        return from_cuda(cudaGetLastError());
    }
    // fused: the d_v / NVD blocks of one head form a cluster along y when the
    // epilogue needs the whole row
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = (fz->gate != nullptr) ? (unsigned)(d_v / NVD) : 1u;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return from_cuda(cudaLaunchKernelEx(&cfg, decode_step_kernel<IO, DK, NVD, true>, static_cast<const IO *>(q),
                                        static_cast<const IO *>(k), static_cast<const IO *>(v),
                                        static_cast<const IO *>(la), static_cast<const IO *>(b),
                                        static_cast<const IO *>(w), S, static_cast<IO *>(o), d_v, H, HV, *fz));
}

// Checks the fusion arguments of the _ex entry points and fills `fz`.
gdn2_status_t check_fuse(int flags, float l2_eps, const void *gate, const float *norm_weight, float norm_eps,
                         FuseArgs *fz) {
    if (flags & ~(GDN2_FUSE_INPUT_PREP | GDN2_FUSE_NEG_EIGVAL)) return GDN2_ERR_INVALID_ARG;
    if ((flags & GDN2_FUSE_NEG_EIGVAL) && !(flags & GDN2_FUSE_INPUT_PREP)) return GDN2_ERR_INVALID_ARG;
    if ((flags & GDN2_FUSE_INPUT_PREP) && !(l2_eps >= 0.f)) return GDN2_ERR_INVALID_ARG;
    if (gate != nullptr && (norm_weight == nullptr || !(norm_eps >= 0.f))) return GDN2_ERR_INVALID_ARG;
    if ((gate && !aligned16(gate)) || (norm_weight && !aligned16(norm_weight))) return GDN2_ERR_MISALIGNED;
    fz->prep = (flags & GDN2_FUSE_INPUT_PREP) ? 1 : 0;
    fz->neg_eigval = (flags & GDN2_FUSE_NEG_EIGVAL) ? 1 : 0;
    fz->l2_eps = l2_eps;
    fz->gate = gate;
    fz->norm_weight = gate ? norm_weight : nullptr;
    fz->norm_eps = norm_eps;
    return GDN2_OK;
}

// Shared validation of the chunk entry points.
gdn2_status_t check_chunk(const void *q, const void *k, const void *v, const void *la, const void *b,
                          const void *w, const float *S0, void *o, float *S_T, const Shape &sh, int chunk,
                          gdn2_io_t io) {
    const int B = sh.B, T = sh.T, H = sh.H, HV = sh.HV, d_k = sh.d_k, d_v = sh.d_v;
    // With T = 0 the token tensors are empty and may be null.
    if (T > 0 && (!q || !k || !v || !la || !b || !w || !o)) return GDN2_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || HV <= 0 || T < 0 || d_k <= 0 || d_v <= 0 || chunk <= 0) return GDN2_ERR_INVALID_ARG;
    if (HV % H != 0) return GDN2_ERR_INVALID_ARG;
    if (io != GDN2_IO_F32 && io != GDN2_IO_BF16) return GDN2_ERR_INVALID_ARG;
    const void *ptrs[9] = {q, k, v, la, b, w, S0, o, S_T};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDN2_ERR_MISALIGNED;
    if (sh.cu && (reinterpret_cast<uintptr_t>(sh.cu) & 3u)) return GDN2_ERR_MISALIGNED;
    if (chunk != 16 && chunk != 32 && chunk != 64) return GDN2_ERR_UNSUPPORTED;
    if (d_k != 64 && d_k != 128) return GDN2_ERR_UNSUPPORTED;
    if (d_v % 64 != 0 || d_v > 512) return GDN2_ERR_UNSUPPORTED;
    if ((long)sh.tensor_b() * T > INT_MAX || B > 65535 || HV > 65535) return GDN2_ERR_UNSUPPORTED;
    return GDN2_OK;
}

// No tokens at all: every final state is its initial state.
gdn2_status_t empty_sequence(const float *S0, float *S_T, const Shape &sh, cudaStream_t st) {
    if (!S_T) return GDN2_OK;
    const size_t bytes = sizeof(float) * (size_t)sh.B * sh.HV * sh.d_k * sh.d_v;
    if (!S0) return from_cuda(cudaMemsetAsync(S_T, 0, bytes, st));
    if (S0 == S_T) return GDN2_OK;
    return from_cuda(cudaMemcpyAsync(S_T, S0, bytes, cudaMemcpyDeviceToDevice, st));
}

template <typename IO>
gdn2_status_t dispatch_ffma_io(const void *q, const void *k, const void *v, const void *la, const void *b,
                               const void *w, const float *S0, void *o, float *S_T, const Shape &sh, int chunk,
                               cudaStream_t st, const FuseArgs *fz) {
#define GDN2_FFMA(DK, CH) return launch_ffma<IO, DK, CH>(q, k, v, la, b, w, S0, o, S_T, sh, st, fz)
    if (sh.d_k == 64) {
        if (chunk == 16) GDN2_FFMA(64, 16);
        if (chunk == 32) GDN2_FFMA(64, 32);
        GDN2_FFMA(64, 64);
    }
    if (chunk == 16) GDN2_FFMA(128, 16);
    if (chunk == 32) GDN2_FFMA(128, 32);
    GDN2_FFMA(128, 64);
#undef GDN2_FFMA
}

gdn2_status_t dispatch_ffma(const void *q, const void *k, const void *v, const void *la, const void *b,
                            const void *w, const float *S0, void *o, float *S_T, const Shape &sh, int chunk,
                            gdn2_io_t io, cudaStream_t st, const FuseArgs *fz = nullptr) {
    gdn2_status_t s = bounds_chunk(q, k, v, la, b, nullptr, w, S0, o, S_T, sh.B, sh.tensor_b(), sh.T, sh.H, sh.HV,
                                   sh.d_k, sh.d_v, sh.cu, io == GDN2_IO_F32 ? 4 : 2, fz, st);
    if (s != GDN2_OK) return s;
    if (io == GDN2_IO_F32) return dispatch_ffma_io<float>(q, k, v, la, b, w, S0, o, S_T, sh, chunk, st, fz);
    return dispatch_ffma_io<__nv_bfloat16>(q, k, v, la, b, w, S0, o, S_T, sh, chunk, st, fz);
}

gdn2_status_t dispatch_tc(const void *q, const void *k, const void *v, const void *la, const void *b,
                          const void *w, const float *S0, void *o, float *S_T, const Shape &sh, cudaStream_t st,
                          const FuseArgs *fz = nullptr) {
    gdn2_status_t s = bounds_chunk(q, k, v, la, b, nullptr, w, S0, o, S_T, sh.B, sh.tensor_b(), sh.T, sh.H, sh.HV,
                                   sh.d_k, sh.d_v, sh.cu, 2, fz, st);
    if (s != GDN2_OK) return s;
    const bool wide = (sh.d_v % 128 == 0);
    if (sh.d_k == 64)
        return wide ? launch_tc<64, 128>(q, k, v, la, b, w, S0, o, S_T, sh, st, fz)
                    : launch_tc<64, 64>(q, k, v, la, b, w, S0, o, S_T, sh, st, fz);
    return wide ? launch_tc<128, 128>(q, k, v, la, b, w, S0, o, S_T, sh, st, fz)
                : launch_tc<128, 64>(q, k, v, la, b, w, S0, o, S_T, sh, st, fz);
}

}  // namespace
}  // namespace gdn2

using namespace gdn2;

extern "C" gdn2_status_t gdn2_chunk_fwd(const void *q, const void *k, const void *v, const void *log_alpha,
                                        const void *b, const void *w, const float *S0, void *o, float *S_T, int B,
                                        int T, int H, int d_k, int d_v, int chunk, gdn2_io_t io, void *stream) {
    const Shape sh{B, T, H, H, d_k, d_v, nullptr};
    gdn2_status_t s = check_chunk(q, k, v, log_alpha, b, w, S0, o, S_T, sh, chunk, io);
    if (s != GDN2_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (T == 0) return empty_sequence(S0, S_T, sh, st);
    if (io == GDN2_IO_F32 || chunk != 64) return dispatch_ffma(q, k, v, log_alpha, b, w, S0, o, S_T, sh, chunk, io, st);
    return dispatch_tc(q, k, v, log_alpha, b, w, S0, o, S_T, sh, st);
}

// ------------------------------------------------ host buffers, pipelined
// The batch is cut into slices of whole sequences.  Slice i is copied in on
// one helper stream, computed on the caller's stream and copied out on a
// second helper stream, so the copy-in of slice i + 1 and the copy-out of
// slice i - 1 run under the kernel of slice i.  Device buffers come from the
// caller's workspace: kHostBufs slice buffers, reused round robin.
namespace {
constexpr int kHostBufs = 2;
constexpr int kHostMaxSlices = 64;
constexpr size_t kHostAlign = 256;

size_t round_up(size_t x) { return (x + kHostAlign - 1) / kHostAlign * kHostAlign; }

// Helper streams and events of the host-buffer entry, created once per device
// and kept for the life of the process (creating streams per call lets them
// alias onto the hardware queues of earlier calls' streams).  `lock` is held
// while a call enqueues its work; an event is re-recorded only after every
// wait on its previous record has been enqueued.
struct HostPipe {
    std::mutex lock;
    bool ready = false;
    cudaStream_t in = nullptr, out = nullptr;
    cudaEvent_t ev0 = nullptr, ev_in[kHostBufs] = {}, ev_k[kHostBufs] = {}, ev_out[kHostBufs] = {};
    cudaEvent_t ev_end_in = nullptr, ev_end_out = nullptr;   // error exit: the helper streams' tails
    cudaError_t init() {
        if (ready) return cudaSuccess;
        cudaError_t e = cudaStreamCreateWithFlags(&in, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&out, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev0, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_end_in, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_end_out, cudaEventDisableTiming);
        for (int i = 0; i < kHostBufs && e == cudaSuccess; ++i) {
            e = cudaEventCreateWithFlags(&ev_in[i], cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_k[i], cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_out[i], cudaEventDisableTiming);
        }
        ready = e == cudaSuccess;
        return e;
    }
};
constexpr int kMaxDevices = 64;
HostPipe g_host_pipes[kMaxDevices];

struct HostSlicing {
    int per, count;            // sequences per slice, number of slices
    size_t key, val, state;    // bytes per sequence: one key tensor, one value tensor, one state
    size_t buffer;             // bytes of one slice buffer
};

HostSlicing host_slicing(int B, int T, int H, int d_k, int d_v, gdn2_io_t io) {
    HostSlicing h;
    const size_t e = io == GDN2_IO_BF16 ? 2 : 4;
    h.count = B < kHostMaxSlices ? B : kHostMaxSlices;
    h.per = (B + h.count - 1) / h.count;
    h.count = (B + h.per - 1) / h.per;
    h.key = (size_t)T * H * d_k * e;
    h.val = (size_t)T * H * d_v * e;
    h.state = (size_t)H * d_k * d_v * sizeof(float);
    // q, k, log_alpha, b; v, w, o; S0, S_T
    h.buffer = 4 * round_up(h.per * h.key) + 3 * round_up(h.per * h.val) + 2 * round_up(h.per * h.state);
    return h;
}
}  // namespace

extern "C" gdn2_status_t gdn2_chunk_fwd_host_workspace(int B, int T, int H, int d_k, int d_v, gdn2_io_t io,
                                                       size_t *bytes) {
    if (!bytes || B <= 0 || T < 0 || H <= 0 || d_k <= 0 || d_v <= 0) return GDN2_ERR_INVALID_ARG;
    if (io != GDN2_IO_F32 && io != GDN2_IO_BF16) return GDN2_ERR_INVALID_ARG;
    const HostSlicing h = host_slicing(B, T, H, d_k, d_v, io);
    *bytes = (h.count < kHostBufs ? h.count : kHostBufs) * h.buffer;
    return GDN2_OK;
}

extern "C" gdn2_status_t gdn2_chunk_fwd_host(const void *q, const void *k, const void *v, const void *log_alpha,
                                             const void *b, const void *w, const float *S0, void *o, float *S_T,
                                             int B, int T, int H, int d_k, int d_v, int chunk, gdn2_io_t io,
                                             void *workspace, size_t workspace_bytes, void *stream) {
    const Shape sh{B, T, H, H, d_k, d_v, nullptr};
    gdn2_status_t s = check_chunk(q, k, v, log_alpha, b, w, S0, o, S_T, sh, chunk, io);
    if (s != GDN2_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const HostSlicing h = host_slicing(B, T, H, d_k, d_v, io);
    if (T == 0) {   // S_T = S0 (or zeros); this case waits for the stream's earlier work
        if (!S_T || S0 == S_T) return GDN2_OK;
        const size_t bytes = (size_t)B * h.state;
        const cudaError_t e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) return from_cuda(e);
        if (S0) memcpy(S_T, S0, bytes);
        else memset(S_T, 0, bytes);
        return GDN2_OK;
    }
    size_t need = 0;
    gdn2_chunk_fwd_host_workspace(B, T, H, d_k, d_v, io, &need);
    if (!workspace || workspace_bytes < need) return GDN2_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) % kHostAlign) return GDN2_ERR_MISALIGNED;

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return from_cuda(e);
    if (dev < 0 || dev >= kMaxDevices) return GDN2_ERR_UNSUPPORTED;
    HostPipe &pp = g_host_pipes[dev];
    std::lock_guard<std::mutex> guard(pp.lock);
    if ((e = pp.init()) != cudaSuccess) return from_cuda(e);
    cudaStream_t sin = pp.in, sout = pp.out;
    cudaEvent_t *ev_in = pp.ev_in, *ev_k = pp.ev_k, *ev_out = pp.ev_out;
    // the helper streams start after the work already on the caller's stream
    e = cudaEventRecord(pp.ev0, st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(sin, pp.ev0, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(sout, pp.ev0, 0);
    if (e != cudaSuccess) return from_cuda(e);
    // An error after this point still leaves the call's work ordered on `st`:
    // the caller's stream waits for whatever the helper streams have queued,
    // so no copy into or out of the workspace outlives the call's stream order.
    auto fail_status = [&](gdn2_status_t status) {
        if (cudaEventRecord(pp.ev_end_in, sin) == cudaSuccess) cudaStreamWaitEvent(st, pp.ev_end_in, 0);
        if (cudaEventRecord(pp.ev_end_out, sout) == cudaSuccess) cudaStreamWaitEvent(st, pp.ev_end_out, 0);
        return status;
    };
    auto fail = [&](cudaError_t err) { return fail_status(from_cuda(err)); };

    const char *hq = static_cast<const char *>(q), *hk = static_cast<const char *>(k);
    const char *hla = static_cast<const char *>(log_alpha), *hb = static_cast<const char *>(b);
    const char *hv = static_cast<const char *>(v), *hw = static_cast<const char *>(w);
    const char *hs0 = reinterpret_cast<const char *>(S0);
    char *ho = static_cast<char *>(o), *hst = reinterpret_cast<char *>(S_T);
    for (int i = 0; i < h.count; ++i) {
        const int r = i % kHostBufs, b0 = i * h.per, nb = (B - b0 < h.per) ? B - b0 : h.per;
        char *base = static_cast<char *>(workspace) + (size_t)r * h.buffer;
        char *dq = base, *dk = dq + round_up(h.per * h.key), *dla = dk + round_up(h.per * h.key);
        char *db = dla + round_up(h.per * h.key), *dv = db + round_up(h.per * h.key);
        char *dw = dv + round_up(h.per * h.val), *dout = dw + round_up(h.per * h.val);
        char *ds0 = dout + round_up(h.per * h.val), *dsT = ds0 + round_up(h.per * h.state);
        const size_t kb = nb * h.key, vb = nb * h.val, sbytes = nb * h.state;
        const size_t ko = b0 * h.key, vo = b0 * h.val, so = b0 * h.state;
        // copy in, once the kernel that last read this buffer is done
        if (i >= kHostBufs && (e = cudaStreamWaitEvent(sin, ev_k[r], 0)) != cudaSuccess) return fail(e);
        const void *src[6] = {hq + ko, hk + ko, hla + ko, hb + ko, hv + vo, hw + vo};
        void *dst[6] = {dq, dk, dla, db, dv, dw};
        const size_t len[6] = {kb, kb, kb, kb, vb, vb};
        for (int j = 0; j < 6 && e == cudaSuccess; ++j)
            e = cudaMemcpyAsync(dst[j], src[j], len[j], cudaMemcpyHostToDevice, sin);
        if (e == cudaSuccess && S0) e = cudaMemcpyAsync(ds0, hs0 + so, sbytes, cudaMemcpyHostToDevice, sin);
        if (e == cudaSuccess) e = cudaEventRecord(ev_in[r], sin);
        // compute, once the inputs are in and the previous outputs of this buffer are out
        if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ev_in[r], 0);
        if (e == cudaSuccess && i >= kHostBufs) e = cudaStreamWaitEvent(st, ev_out[r], 0);
        if (e != cudaSuccess) return fail(e);
        const Shape ssh{nb, T, H, H, d_k, d_v, nullptr};
        const float *s0p = S0 ? reinterpret_cast<const float *>(ds0) : nullptr;
        float *stp = S_T ? reinterpret_cast<float *>(dsT) : nullptr;
        s = (io == GDN2_IO_F32 || chunk != 64)
                ? dispatch_ffma(dq, dk, dv, dla, db, dw, s0p, dout, stp, ssh, chunk, io, st)
                : dispatch_tc(dq, dk, dv, dla, db, dw, s0p, dout, stp, ssh, st);
        if (s != GDN2_OK) return fail_status(s);
        // copy out
        if ((e = cudaEventRecord(ev_k[r], st)) != cudaSuccess) return fail(e);
        if ((e = cudaStreamWaitEvent(sout, ev_k[r], 0)) != cudaSuccess) return fail(e);
        e = cudaMemcpyAsync(ho + vo, dout, vb, cudaMemcpyDeviceToHost, sout);
        if (e == cudaSuccess && S_T) e = cudaMemcpyAsync(hst + so, dsT, sbytes, cudaMemcpyDeviceToHost, sout);
        if (e == cudaSuccess) e = cudaEventRecord(ev_out[r], sout);
        if (e != cudaSuccess) return fail(e);
    }
    // the caller's stream ends after the last copy out
    return from_cuda(cudaStreamWaitEvent(st, ev_out[(h.count - 1) % kHostBufs], 0));
}

extern "C" gdn2_status_t gdn2_chunk_fwd_ex(const void *q, const void *k, const void *v, const void *log_alpha,
                                           const void *b, const void *w, const float *S0, void *o, float *S_T,
                                           int B, int T, int H, int HV, int d_k, int d_v, int chunk, gdn2_io_t io,
                                           const int *cu_seqlens, int flags, float l2_eps, const void *gate,
                                           const float *norm_weight, float norm_eps, void *stream) {
    FuseArgs fz;
    gdn2_status_t s = check_fuse(flags, l2_eps, gate, norm_weight, norm_eps, &fz);
    if (s != GDN2_OK) return s;
    const Shape sh{B, T, H, HV != 0 ? HV : H, d_k, d_v, cu_seqlens};
    s = check_chunk(q, k, v, log_alpha, b, w, S0, o, S_T, sh, chunk, io);
    if (s != GDN2_OK) return s;
    if (gate == nullptr && norm_weight != nullptr) return GDN2_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (T == 0) return empty_sequence(S0, S_T, sh, st);
    if (io == GDN2_IO_F32 || chunk != 64)
        return dispatch_ffma(q, k, v, log_alpha, b, w, S0, o, S_T, sh, chunk, io, st, &fz);
    return dispatch_tc(q, k, v, log_alpha, b, w, S0, o, S_T, sh, st, &fz);
}

extern "C" gdn2_status_t gdn2_chunk_fwd_cuda_core(const void *q, const void *k, const void *v,
                                                  const void *log_alpha, const void *b, const void *w,
                                                  const float *S0, void *o, float *S_T, int B, int T, int H,
                                                  int d_k, int d_v, int chunk, gdn2_io_t io, void *stream) {
    const Shape sh{B, T, H, H, d_k, d_v, nullptr};
    gdn2_status_t s = check_chunk(q, k, v, log_alpha, b, w, S0, o, S_T, sh, chunk, io);
    if (s != GDN2_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (T == 0) return empty_sequence(S0, S_T, sh, st);
    return dispatch_ffma(q, k, v, log_alpha, b, w, S0, o, S_T, sh, chunk, io, st);
}

namespace gdn2 {
namespace {
gdn2_status_t decode_impl(const void *q, const void *k, const void *v, const void *log_alpha, const void *b,
                          const void *w, float *S, void *o, int B, int H, int HV, int d_k, int d_v, gdn2_io_t io,
                          void *stream, const FuseArgs *fz) {
    if (!q || !k || !v || !log_alpha || !b || !w || !S || !o) return GDN2_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || HV <= 0 || d_k <= 0 || d_v <= 0) return GDN2_ERR_INVALID_ARG;
    if (HV % H != 0) return GDN2_ERR_INVALID_ARG;
    if (io != GDN2_IO_F32 && io != GDN2_IO_BF16) return GDN2_ERR_INVALID_ARG;
    const void *ptrs[8] = {q, k, v, log_alpha, b, w, S, o};
    for (const void *p : ptrs)
        if (!aligned16(p)) return GDN2_ERR_MISALIGNED;
    if (d_k != 64 && d_k != 128) return GDN2_ERR_UNSUPPORTED;
    if (d_v % 64 != 0 || d_v > 512) return GDN2_ERR_UNSUPPORTED;
    if ((long)B * HV > INT_MAX) return GDN2_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool wide = (d_v % 128 == 0);
#define GDN2_DECODE(IO, DK)                                                                            \
    return wide ? launch_decode<IO, DK, 128>(q, k, v, log_alpha, b, w, S, o, B, H, HV, d_v, st, fz)     \
                : launch_decode<IO, DK, 64>(q, k, v, log_alpha, b, w, S, o, B, H, HV, d_v, st, fz)
    if (io == GDN2_IO_F32) {
        if (d_k == 64) GDN2_DECODE(float, 64);
        GDN2_DECODE(float, 128);
    }
    if (d_k == 64) GDN2_DECODE(__nv_bfloat16, 64);
    GDN2_DECODE(__nv_bfloat16, 128);
#undef GDN2_DECODE
}
}  // namespace
}  // namespace gdn2

extern "C" gdn2_status_t gdn2_decode_step(const void *q, const void *k, const void *v, const void *log_alpha,
                                          const void *b, const void *w, float *S, void *o, int B, int H, int d_k,
                                          int d_v, gdn2_io_t io, void *stream) {
    return decode_impl(q, k, v, log_alpha, b, w, S, o, B, H, H, d_k, d_v, io, stream, nullptr);
}

extern "C" gdn2_status_t gdn2_decode_step_ex(const void *q, const void *k, const void *v, const void *log_alpha,
                                             const void *b, const void *w, float *S, void *o, int B, int H,
                                             int HV, int d_k, int d_v, gdn2_io_t io, int flags, float l2_eps,
                                             const void *gate, const float *norm_weight, float norm_eps,
                                             void *stream) {
    FuseArgs fz;
    const gdn2_status_t s = check_fuse(flags, l2_eps, gate, norm_weight, norm_eps, &fz);
    if (s != GDN2_OK) return s;
    if (gate == nullptr && norm_weight != nullptr) return GDN2_ERR_INVALID_ARG;
    return decode_impl(q, k, v, log_alpha, b, w, S, o, B, H, HV != 0 ? HV : H, d_k, d_v, io, stream, &fz);
}

namespace gdn2 {
namespace {
template <typename IO, int DK>
gdn2_status_t launch_qed_chunk(const void *q, const void *k, const void *v, const void *la, const void *b,
                               const void *c, const void *w, const float *S0, void *o, float *S_T, int B,
                               int T, int H, int d_v, float eps, cudaStream_t st) {
    if (launch_gate() != GDN2_OK) return GDN2_ERR_CUDA;
    using Cfg = QedCfg<DK>;
    auto kern = chunk_fwd_qed_kernel<IO, DK>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::BYTES) != cudaSuccess)
        return GDN2_ERR_CUDA;
    dim3 grid(d_v / Cfg::NV, H, B);
    kern<<<grid, 256, Cfg::BYTES, st>>>(static_cast<const IO *>(q), static_cast<const IO *>(k),
                                        static_cast<const IO *>(v), static_cast<const IO *>(la),
                                        static_cast<const IO *>(b), static_cast<const IO *>(c),
                                        static_cast<const IO *>(w), S0, static_cast<IO *>(o), S_T, T, H, d_v, eps);
    return from_cuda(cudaGetLastError());
}

template <typename IO, int DK, int NVD>
gdn2_status_t launch_qed_decode(const void *q, const void *k, const void *v, const void *la, const void *b,
                                const void *c, const void *w, float *S, void *o, int B, int H, int d_v, float eps,
                                cudaStream_t st) {
    if (launch_gate() != GDN2_OK) return GDN2_ERR_CUDA;
    gdn2_status_t s = bounds_chunk(q, k, v, la, b, c, w, S, o, S, B, B, 1, H, H, DK, d_v, nullptr, sizeof(IO),
                                   nullptr, st);
    if (s != GDN2_OK) return s;
    dim3 grid((unsigned)((long)B * H), d_v / NVD);
    decode_step_qed_kernel<IO, DK, NVD><<<grid, 256, 0, st>>>(
        static_cast<const IO *>(q), static_cast<const IO *>(k), static_cast<const IO *>(v),
        static_cast<const IO *>(la), static_cast<const IO *>(b), static_cast<const IO *>(c),
        static_cast<const IO *>(w), S, static_cast<IO *>(o), d_v, eps);
    return from_cuda(cudaGetLastError());
}
}  // namespace
}  // namespace gdn2

extern "C" gdn2_status_t gdn2_chunk_fwd_qed(const void *q, const void *k, const void *v, const void *log_alpha,
                                            const void *b, const void *c, const void *w, const float *S0, void *o,
                                            float *S_T, int B, int T, int H, int d_k, int d_v, gdn2_io_t io,
                                            float qed_eps, void *stream) {
    const Shape sh{B, T, H, H, d_k, d_v, nullptr};
    gdn2_status_t s = check_chunk(q, k, v, log_alpha, b, w, S0, o, S_T, sh, 64, io);
    if (s != GDN2_OK) return s;
    if (T > 0 && c == nullptr) return GDN2_ERR_INVALID_ARG;
    if (!(qed_eps >= 0.f)) return GDN2_ERR_INVALID_ARG;
    if (c && !aligned16(c)) return GDN2_ERR_MISALIGNED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (T == 0) return empty_sequence(S0, S_T, sh, st);
    s = bounds_chunk(q, k, v, log_alpha, b, c, w, S0, o, S_T, B, B, T, H, H, d_k, d_v, nullptr,
                     io == GDN2_IO_F32 ? 4 : 2, nullptr, st);
    if (s != GDN2_OK) return s;
    if (io == GDN2_IO_F32) {
        if (d_k == 64) return launch_qed_chunk<float, 64>(q, k, v, log_alpha, b, c, w, S0, o, S_T, B, T, H, d_v, qed_eps, st);
        return launch_qed_chunk<float, 128>(q, k, v, log_alpha, b, c, w, S0, o, S_T, B, T, H, d_v, qed_eps, st);
    }
    // bf16 I/O: the tensor-core kernel
    const bool wide = (d_v % 128 == 0);
    if (d_k == 64)
        return wide ? launch_tc_qed<64, 128>(q, k, v, log_alpha, b, c, w, S0, o, S_T, B, T, H, d_v, qed_eps, st)
                    : launch_tc_qed<64, 64>(q, k, v, log_alpha, b, c, w, S0, o, S_T, B, T, H, d_v, qed_eps, st);
    return wide ? launch_tc_qed<128, 128>(q, k, v, log_alpha, b, c, w, S0, o, S_T, B, T, H, d_v, qed_eps, st)
                : launch_tc_qed<128, 64>(q, k, v, log_alpha, b, c, w, S0, o, S_T, B, T, H, d_v, qed_eps, st);
}

extern "C" gdn2_status_t gdn2_decode_step_qed(const void *q, const void *k, const void *v, const void *log_alpha,
                                              const void *b, const void *c, const void *w, float *S, void *o,
                                              int B, int H, int d_k, int d_v, gdn2_io_t io, float qed_eps,
                                              void *stream) {
    if (!q || !k || !v || !log_alpha || !b || !c || !w || !S || !o) return GDN2_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || d_k <= 0 || d_v <= 0 || !(qed_eps >= 0.f)) return GDN2_ERR_INVALID_ARG;
    if (io != GDN2_IO_F32 && io != GDN2_IO_BF16) return GDN2_ERR_INVALID_ARG;
    const void *ptrs[9] = {q, k, v, log_alpha, b, c, w, S, o};
    for (const void *p : ptrs)
        if (!aligned16(p)) return GDN2_ERR_MISALIGNED;
    if (d_k != 64 && d_k != 128) return GDN2_ERR_UNSUPPORTED;
    if (d_v % 64 != 0 || d_v > 512) return GDN2_ERR_UNSUPPORTED;
    if ((long)B * H > INT_MAX) return GDN2_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool wide = (d_v % 128 == 0);
#define GDN2_QED_DECODE(IO, DK)                                                                                  \
    return wide ? launch_qed_decode<IO, DK, 128>(q, k, v, log_alpha, b, c, w, S, o, B, H, d_v, qed_eps, st)     \
                : launch_qed_decode<IO, DK, 64>(q, k, v, log_alpha, b, c, w, S, o, B, H, d_v, qed_eps, st)
    if (io == GDN2_IO_F32) {
        if (d_k == 64) GDN2_QED_DECODE(float, 64);
        GDN2_QED_DECODE(float, 128);
    }
    if (d_k == 64) GDN2_QED_DECODE(__nv_bfloat16, 64);
    GDN2_QED_DECODE(__nv_bfloat16, 128);
#undef GDN2_QED_DECODE
}

extern "C" gdn2_status_t gdn2_device_status(void *stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return GDN2_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return GDN2_ERR_CUDA;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return GDN2_ERR_CUDA;
        return static_cast<gdn2_status_t>(v);
    }
    return GDN2_OK;
}

extern "C" gdn2_status_t gdn2_selftest_wait_timeout(int limit_us, void *stream) {
    if (limit_us < 1 || limit_us > 1000000) return GDN2_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    selftest_wait_kernel<<<1, 32, 0, st>>>(1000ull * (unsigned long long)limit_us);
    if (cudaGetLastError() != cudaSuccess) return GDN2_ERR_CUDA;
    return gdn2_device_status(stream);
}

extern "C" gdn2_status_t gdn2_testing_fail_launches(int pass, int fail) {
    if (pass < 0 || fail < 0) return GDN2_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> guard(g_inject_lock);
    g_inject_pass = pass;
    g_inject_fail = fail;
    g_inject_armed.store(fail > 0, std::memory_order_relaxed);
    return GDN2_OK;
}

extern "C" gdn2_status_t gdn2_debug_bounds_site(int *buffer, int *line, void *stream) {
    if (!buffer || !line) return GDN2_ERR_INVALID_ARG;
    *buffer = -1;
    *line = 0;
#ifdef GDN2_DEBUG_BOUNDS
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return GDN2_ERR_CUDA;
    unsigned int v = 0u;
    if (cudaMemcpyFromSymbol(&v, g_bounds_site, sizeof(v)) != cudaSuccess) return GDN2_ERR_CUDA;
    if (v != 0u) {
        const unsigned int zero = 0u;
        if (cudaMemcpyToSymbol(g_bounds_site, &zero, sizeof(zero)) != cudaSuccess) return GDN2_ERR_CUDA;
        *buffer = (int)(v >> 16) - 1;
        *line = (int)(v & 0xffffu);
    }
    return GDN2_OK;
#else
    (void)stream;
    return GDN2_ERR_UNSUPPORTED;
#endif
}

extern "C" gdn2_status_t gdn2_selftest_bounds(void *stream) {
#ifdef GDN2_DEBUG_BOUNDS
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    selftest_bounds_kernel<<<1, 1, 0, st>>>(1ull << 40);
    if (cudaGetLastError() != cudaSuccess) return GDN2_ERR_CUDA;
    return gdn2_device_status(stream);
#else
    (void)stream;
    return GDN2_ERR_UNSUPPORTED;
#endif
}

extern "C" const char *gdn2_status_string(gdn2_status_t status) {
    switch (status) {
        case GDN2_OK: return "GDN2_OK";
        case GDN2_ERR_INVALID_ARG: return "GDN2_ERR_INVALID_ARG";
        case GDN2_ERR_UNSUPPORTED: return "GDN2_ERR_UNSUPPORTED";
        case GDN2_ERR_MISALIGNED: return "GDN2_ERR_MISALIGNED";
        case GDN2_ERR_CUDA: return "GDN2_ERR_CUDA";
        case GDN2_ERR_DEVICE_TIMEOUT: return "GDN2_ERR_DEVICE_TIMEOUT";
        case GDN2_ERR_OUT_OF_BOUNDS: return "GDN2_ERR_OUT_OF_BOUNDS";
        default: return "GDN2_ERR_UNKNOWN";
    }
}

extern "C" int gdn2_version(void) { return 100; }
