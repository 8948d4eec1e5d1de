"""Python binding of the sm_100a Gated DeltaNet-2 library (``libgdn2.so``).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI of ``include/gdn2.h``.  torch supplies device
memory and the stream; there is no CPU path and no fallback.  If the
library has not been built this module raises on first use.

    chunk_fwd(q, k, v, log_alpha, b, w, S0=None) -> (o, S_T)
    decode_step(q, k, v, log_alpha, b, w, S)     -> o      (S updated in place)
    chunk_fwd_qed / decode_step_qed              -- with the second, query-derived
        erase direction (gate c on the key axis)
    chunk_fwd_ex / decode_step_ex                 -- the same with value heads,
        packed sequences (cu_seqlens, chunk only) and the fused input prep and
        gated RMS-norm output epilogue

Token tensors are [B, T, H, d] (decode: [B, H, d]) in bfloat16 or float32,
contiguous, on one CUDA device; states are float32 [B, HV, d_k, d_v].  q, k,
log_alpha, b carry the H key heads, v, w, o, gate the HV value heads
(HV = H unless the _ex calls are given more value heads).
"""
from __future__ import annotations

import contextlib
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdn2.so")
# the same sources with device-side range checks (-DGDN2_DEBUG_BOUNDS); used in
# place of LIB_PATH when GDN2_DEBUG_BOUNDS=1 is set, or inside debug_bounds()
DEBUG_LIB_PATH = os.path.join(_HERE, "libgdn2_debug.so")

IO_F32 = 0
IO_BF16 = 1
STATUS_NAMES = {0: "GDN2_OK", 1: "GDN2_ERR_INVALID_ARG", 2: "GDN2_ERR_UNSUPPORTED",
                3: "GDN2_ERR_MISALIGNED", 4: "GDN2_ERR_CUDA", 5: "GDN2_ERR_DEVICE_TIMEOUT",
                6: "GDN2_ERR_OUT_OF_BOUNDS"}
OUT_OF_BOUNDS = 6
# argument buffers as gdn2_debug_bounds_site numbers them
BOUNDS_BUFFERS = ("q", "k", "v", "log_alpha", "b", "w", "c", "S0", "S_T", "o", "gate", "norm_weight",
                  "cu_seqlens")
EXPORTED = ("gdn2_chunk_fwd", "gdn2_chunk_fwd_cuda_core", "gdn2_chunk_fwd_host",
            "gdn2_chunk_fwd_host_workspace", "gdn2_chunk_fwd_host_noalloc", "gdn2_decode_step",
            "gdn2_chunk_fwd_ex", "gdn2_decode_step_ex", "gdn2_chunk_fwd_qed", "gdn2_decode_step_qed",
            "gdn2_device_status", "gdn2_selftest_wait_timeout", "gdn2_debug_bounds_site",
            "gdn2_selftest_bounds", "gdn2_testing_fail_launches", "gdn2_status_string", "gdn2_version")
FUSE_INPUT_PREP = 1    # q, k, b, w are raw: L2-normalise q, k over d_k; b, w = sigmoid
FUSE_NEG_EIGVAL = 2    # with FUSE_INPUT_PREP: b = 2 sigmoid(b)
NOALLOC_WORKSPACE_BYTES = 64 << 20   # GDN2_NOALLOC_WORKSPACE_BYTES: the no-alloc entry's fixed workspace

_lib = None
_opened = {}


class Gdn2Error(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = int(status)
        super().__init__(f"{what}: {STATUS_NAMES.get(self.status, self.status)}")


def lib() -> ctypes.CDLL:
    """The library the calls go through: libgdn2.so, or its debug build when
    GDN2_DEBUG_BOUNDS=1 is set (raises if the file is missing)."""
    global _lib
    if _lib is None:
        _lib = _open(DEBUG_LIB_PATH if os.environ.get("GDN2_DEBUG_BOUNDS") == "1" else LIB_PATH)
    return _lib


@contextlib.contextmanager
def debug_bounds():
    """Route the calls made inside the block through the debug build
    (libgdn2_debug.so: every per-thread global access range-checked against its
    argument buffer; a failed check records GDN2_ERR_OUT_OF_BOUNDS instead of
    touching memory).  Yields the debug library."""
    global _lib
    prev = _lib
    _lib = _open(DEBUG_LIB_PATH)
    try:
        yield _lib
    finally:
        _lib = prev


def _open(path: str) -> ctypes.CDLL:
    """Open one build of the library (once) and declare the C signatures."""
    if path not in _opened:
        if not os.path.exists(path):
            raise ImportError(f"{path} is missing: build it with "
                              "`python -m gated_delta_rule_92_b200.build`")
        L = ctypes.CDLL(path)
        P, I = ctypes.c_void_p, ctypes.c_int
        chunk_args = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, P]
        for name in ("gdn2_chunk_fwd", "gdn2_chunk_fwd_cuda_core"):
            getattr(L, name).argtypes = chunk_args
            getattr(L, name).restype = I
        # (..., B, T, H, d_k, d_v, chunk, io, workspace, workspace_bytes, stream)
        L.gdn2_chunk_fwd_host.argtypes = chunk_args[:-1] + [P, ctypes.c_size_t, P]
        L.gdn2_chunk_fwd_host.restype = I
        L.gdn2_chunk_fwd_host_workspace.argtypes = [I] * 6 + [ctypes.POINTER(ctypes.c_size_t)]
        L.gdn2_chunk_fwd_host_workspace.restype = I
        L.gdn2_chunk_fwd_host_noalloc.argtypes = chunk_args
        L.gdn2_chunk_fwd_host_noalloc.restype = I
        L.gdn2_decode_step.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, P]
        L.gdn2_decode_step.restype = I
        F = ctypes.c_float
        fuse_args = [I, F, P, P, F]
        # (..., B, T, H, HV, d_k, d_v, chunk, io, cu_seqlens, flags, l2_eps, gate, weight, eps, stream)
        L.gdn2_chunk_fwd_ex.argtypes = [P] * 9 + [I] * 8 + [P] + fuse_args + [P]
        L.gdn2_chunk_fwd_ex.restype = I
        # (..., B, H, HV, d_k, d_v, io, flags, l2_eps, gate, weight, eps, stream)
        L.gdn2_decode_step_ex.argtypes = [P] * 8 + [I] * 6 + fuse_args + [P]
        L.gdn2_decode_step_ex.restype = I
        # (q, k, v, log_alpha, b, c, w, S0, o, S_T, B, T, H, d_k, d_v, io, qed_eps, stream)
        L.gdn2_chunk_fwd_qed.argtypes = [P] * 10 + [I] * 6 + [F, P]
        L.gdn2_chunk_fwd_qed.restype = I
        # (q, k, v, log_alpha, b, c, w, S, o, B, H, d_k, d_v, io, qed_eps, stream)
        L.gdn2_decode_step_qed.argtypes = [P] * 9 + [I] * 5 + [F, P]
        L.gdn2_decode_step_qed.restype = I
        L.gdn2_device_status.argtypes = [P]
        L.gdn2_device_status.restype = I
        L.gdn2_selftest_wait_timeout.argtypes = [I, P]
        L.gdn2_selftest_wait_timeout.restype = I
        L.gdn2_status_string.argtypes = [I]
        L.gdn2_status_string.restype = ctypes.c_char_p
        L.gdn2_debug_bounds_site.argtypes = [ctypes.POINTER(I), ctypes.POINTER(I), P]
        L.gdn2_debug_bounds_site.restype = I
        L.gdn2_selftest_bounds.argtypes = [P]
        L.gdn2_selftest_bounds.restype = I
        L.gdn2_testing_fail_launches.argtypes = [I, I]
        L.gdn2_testing_fail_launches.restype = I
        L.gdn2_version.argtypes = []
        L.gdn2_version.restype = I
        _opened[path] = L
    return _opened[path]


def status_string(code: int) -> str:
    return lib().gdn2_status_string(int(code)).decode()


def _io(dtype) -> int:
    if dtype == torch.bfloat16:
        return IO_BF16
    if dtype == torch.float32:
        return IO_F32
    raise TypeError(f"unsupported I/O dtype {dtype}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check_tokens(ts, dtype, device):
    for t in ts:
        if not t.is_cuda or t.device != device:
            raise ValueError("all tensors must be on the same CUDA device")
        if t.dtype != dtype:
            raise TypeError("token tensors must share one dtype")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def _check_state(S, shape, device):
    if S is None:
        return
    if S.dtype != torch.float32 or tuple(S.shape) != tuple(shape) or not S.is_contiguous() \
            or S.device != device:
        raise ValueError(f"state must be contiguous float32 {tuple(shape)} on {device}")


def _fuse_args(q, prep, allow_neg_eigval, l2_eps, gate, norm_weight, norm_eps, gate_shape):
    """The fusion arguments of the _ex calls, checked and marshalled."""
    flags = (FUSE_INPUT_PREP if prep else 0) | (FUSE_NEG_EIGVAL if (prep and allow_neg_eigval) else 0)
    if allow_neg_eigval and not prep:
        raise ValueError("allow_neg_eigval applies to the fused input prep (prep=True)")
    if gate is not None:
        _check_tokens((gate,), q.dtype, q.device)
        if tuple(gate.shape) != tuple(gate_shape):
            raise ValueError(f"gate must be {tuple(gate_shape)}")
        if norm_weight is None or norm_weight.dtype != torch.float32 or not norm_weight.is_contiguous() \
                or tuple(norm_weight.shape) != (gate_shape[-1],) or norm_weight.device != q.device:
            raise ValueError("norm_weight must be a contiguous float32 [d_v] tensor on the device")
    elif norm_weight is not None:
        raise ValueError("norm_weight is only used with gate")
    return [int(flags), ctypes.c_float(float(l2_eps)), _ptr(gate),
            _ptr(norm_weight) if gate is not None else None, ctypes.c_float(float(norm_eps))]


def _chunk(fn_name, q, k, v, log_alpha, b, w, S0, o, S_T, chunk, stream, want_state, fuse=None,
           cu_seqlens=None, ex=False):
    Bt, T, H, dk = q.shape
    HV, dv = v.shape[2], v.shape[3]
    dev = q.device
    _check_tokens((q, k, v, log_alpha, b, w), q.dtype, dev)
    for t in (k, log_alpha, b):
        if tuple(t.shape) != (Bt, T, H, dk):
            raise ValueError("q, k, log_alpha, b must be [B, T, H, d_k]")
    if tuple(v.shape[:2]) != (Bt, T) or tuple(w.shape) != (Bt, T, HV, dv):
        raise ValueError("v, w must be [B, T, HV, d_v]")
    if HV != H and not ex:
        raise ValueError(f"{fn_name} takes H value heads; use chunk_fwd_ex for num_v_heads != H")
    if HV % H != 0:
        raise ValueError("the number of value heads must be a multiple of the key heads")
    B = Bt
    if cu_seqlens is not None:
        if Bt != 1:
            raise ValueError("with cu_seqlens the token tensors are [1, T_total, heads, d]")
        if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2 \
                or cu_seqlens.device != dev or not cu_seqlens.is_contiguous():
            raise ValueError("cu_seqlens must be a contiguous int32 [B + 1] tensor on the device")
        B = cu_seqlens.numel() - 1
    _check_state(S0, (B, HV, dk, dv), dev)
    if o is None:
        o = torch.empty((Bt, T, HV, dv), dtype=q.dtype, device=dev)
    if S_T is None and want_state:
        S_T = torch.empty((B, HV, dk, dv), dtype=torch.float32, device=dev)
    _check_tokens((o,), q.dtype, dev)
    if tuple(o.shape) != (Bt, T, HV, dv):
        raise ValueError(f"o must be {(Bt, T, HV, dv)}")
    _check_state(S_T, (B, HV, dk, dv), dev)
    with torch.cuda.device(dev):
        if ex:
            args = [_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(S0), _ptr(o),
                    _ptr(S_T), B, T, H, HV, dk, dv, int(chunk), _io(q.dtype), _ptr(cu_seqlens)]
            args += fuse(q, (Bt, T, HV, dv))
        else:
            args = [_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w),
                    _ptr(S0), _ptr(o), _ptr(S_T), B, T, H, dk, dv, int(chunk), _io(q.dtype)]
        st = getattr(lib(), fn_name)(*args, _stream(stream))
    if st != 0:
        raise Gdn2Error(st, fn_name)
    return o, S_T


def chunk_fwd(q, k, v, log_alpha, b, w, S0=None, *, o=None, S_T=None, chunk: int = 64,
              stream=None, want_state: bool = True):
    """Chunk-parallel forward; returns (o [B,T,H,d_v], S_T [B,H,d_k,d_v] or None)."""
    return _chunk("gdn2_chunk_fwd", q, k, v, log_alpha, b, w, S0, o, S_T, chunk, stream, want_state)


def chunk_fwd_host_workspace_bytes(B: int, T: int, H: int, d_k: int, d_v: int, dtype) -> int:
    """Device workspace bytes that chunk_fwd_host needs for this shape."""
    n = ctypes.c_size_t(0)
    st = lib().gdn2_chunk_fwd_host_workspace(int(B), int(T), int(H), int(d_k), int(d_v), _io(dtype),
                                             ctypes.byref(n))
    if st != 0:
        raise Gdn2Error(st, "gdn2_chunk_fwd_host_workspace")
    return int(n.value)


def chunk_fwd_host(q, k, v, log_alpha, b, w, S0=None, *, o=None, S_T=None, workspace=None,
                   chunk: int = 64, stream=None, want_state: bool = True):
    """chunk_fwd on HOST (CPU) tensors: the library copies each slice of whole
    sequences in, runs it and copies it out, overlapping the three.  Host
    tensors should be pinned for the copies to overlap.  `workspace` is a
    CUDA uint8 tensor of at least chunk_fwd_host_workspace_bytes (allocated on
    the current device if None).  Returns (o, S_T) as CPU tensors, valid once
    the stream has been synchronised."""
    B, T, H, dk = q.shape
    dv = v.shape[3]
    for t in (q, k, v, log_alpha, b, w):
        if t.is_cuda or t.dtype != q.dtype or not t.is_contiguous():
            raise ValueError("token tensors must be contiguous CPU tensors of one dtype")
    for t in (k, log_alpha, b):
        if tuple(t.shape) != (B, T, H, dk):
            raise ValueError("q, k, log_alpha, b must be [B, T, H, d_k]")
    if tuple(v.shape) != (B, T, H, dv) or tuple(w.shape) != (B, T, H, dv):
        raise ValueError("v, w must be [B, T, H, d_v]")
    pin = q.is_pinned()
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=q.dtype, pin_memory=pin)
    if S_T is None and want_state:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, pin_memory=pin)
    for S in (S0, S_T):
        if S is not None and (S.is_cuda or S.dtype != torch.float32 or not S.is_contiguous()
                              or tuple(S.shape) != (B, H, dk, dv)):
            raise ValueError(f"states must be contiguous float32 CPU tensors {(B, H, dk, dv)}")
    if o.is_cuda or o.dtype != q.dtype or not o.is_contiguous() or tuple(o.shape) != (B, T, H, dv):
        raise ValueError(f"o must be a contiguous CPU tensor {(B, T, H, dv)}")
    need = chunk_fwd_host_workspace_bytes(B, T, H, dk, dv, q.dtype)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device="cuda")
    if not workspace.is_cuda or workspace.dtype != torch.uint8 or workspace.numel() < need:
        raise ValueError(f"workspace must be a CUDA uint8 tensor of at least {need} bytes")
    if stream is not None:
        if stream.device != workspace.device:
            raise ValueError(f"stream is on {stream.device} but the workspace is on {workspace.device}")
        workspace.record_stream(stream)
    with torch.cuda.device(workspace.device):
        st = lib().gdn2_chunk_fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(S0),
                                       _ptr(o), _ptr(S_T), B, T, H, dk, dv, int(chunk), _io(q.dtype),
                                       _ptr(workspace), ctypes.c_size_t(workspace.numel()), _stream(stream))
    if st != 0:
        raise Gdn2Error(st, "gdn2_chunk_fwd_host")
    return o, S_T


def chunk_fwd_host_noalloc(q, k, v, log_alpha, b, w, S0, o, S_T=None, *, chunk: int = 64, stream=None):
    """chunk_fwd_host for callers that cannot allocate device memory: the
    library stages the slices in its own fixed 64 MiB device array instead of
    a caller workspace, and this wrapper allocates nothing either (o and S_T
    are the caller's CPU tensors; S0 and S_T may be None).  Shapes that need
    more than that array raise ValueError.  The first call on a device sets
    the array up, so make it before any stream capture; calls that can
    overlap on the GPU (different streams, unordered) race on the shared
    array.  Returns (o, S_T), valid once the stream has been synchronised."""
    B, T, H, dk = q.shape
    dv = v.shape[3]
    for t in (q, k, v, log_alpha, b, w, o):
        if t.is_cuda or t.dtype != q.dtype or not t.is_contiguous():
            raise ValueError("token tensors and o must be contiguous CPU tensors of one dtype")
    for t in (k, log_alpha, b):
        if tuple(t.shape) != (B, T, H, dk):
            raise ValueError("q, k, log_alpha, b must be [B, T, H, d_k]")
    for t in (v, w, o):
        if tuple(t.shape) != (B, T, H, dv):
            raise ValueError("v, w, o must be [B, T, H, d_v]")
    for S in (S0, S_T):
        if S is not None and (S.is_cuda or S.dtype != torch.float32 or not S.is_contiguous()
                              or tuple(S.shape) != (B, H, dk, dv)):
            raise ValueError(f"states must be contiguous float32 CPU tensors {(B, H, dk, dv)}")
    need = chunk_fwd_host_workspace_bytes(B, T, H, dk, dv, q.dtype)
    if need > NOALLOC_WORKSPACE_BYTES:
        raise ValueError(f"this shape needs a {need}-byte workspace, more than the no-alloc entry's "
                         f"{NOALLOC_WORKSPACE_BYTES} bytes: use chunk_fwd_host with a workspace")
    dev = stream.device if stream is not None else torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(dev):
        st = lib().gdn2_chunk_fwd_host_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w),
                                               _ptr(S0), _ptr(o), _ptr(S_T), B, T, H, dk, dv, int(chunk),
                                               _io(q.dtype), _stream(stream))
    if st != 0:
        raise Gdn2Error(st, "gdn2_chunk_fwd_host_noalloc")
    return o, S_T


def chunk_fwd_ex(q, k, v, log_alpha, b, w, S0=None, *, cu_seqlens=None, prep: bool = False,
                 allow_neg_eigval: bool = False, l2_eps: float = 1e-6, gate=None, norm_weight=None,
                 norm_eps: float = 1e-5, o=None, S_T=None, chunk: int = 64, stream=None,
                 want_state: bool = True):
    """Chunk forward, generalised and fused:

    * value heads: v, w (and gate, o) may carry HV = G * H heads; value head hv
      reads key head hv // G.  States are [B, HV, d_k, d_v].
    * cu_seqlens: int32 [B + 1] device offsets of B sequences packed along T;
      token tensors are then [1, T_total, heads, d].
    * prep=True: q, k, b, w are raw (L2-normalised / sigmoid in the kernel);
      allow_neg_eigval doubles b.
    * gate [.., HV, d_v] with norm_weight [d_v] fp32: the gated RMS-norm output
      epilogue.

    Returns (o or y, S_T)."""
    fuse = lambda q_, shape: _fuse_args(q_, prep, allow_neg_eigval, l2_eps, gate, norm_weight,
                                        norm_eps, shape)
    return _chunk("gdn2_chunk_fwd_ex", q, k, v, log_alpha, b, w, S0, o, S_T, chunk, stream,
                  want_state, fuse, cu_seqlens=cu_seqlens, ex=True)


def chunk_fwd_cuda_core(q, k, v, log_alpha, b, w, S0=None, *, o=None, S_T=None, chunk: int = 64,
                        stream=None, want_state: bool = True):
    """The same forward on the CUDA-core (fp32 FFMA) chunk kernel."""
    return _chunk("gdn2_chunk_fwd_cuda_core", q, k, v, log_alpha, b, w, S0, o, S_T, chunk, stream,
                  want_state)


def _decode(fn_name, q, k, v, log_alpha, b, w, S, o, stream, fuse=None, ex=False):
    B, H, dk = q.shape
    HV, dv = v.shape[1], v.shape[2]
    dev = q.device
    _check_tokens((q, k, v, log_alpha, b, w), q.dtype, dev)
    for t in (k, log_alpha, b):
        if tuple(t.shape) != (B, H, dk):
            raise ValueError("q, k, log_alpha, b must be [B, H, d_k]")
    if v.shape[0] != B or tuple(w.shape) != (B, HV, dv):
        raise ValueError("v, w must be [B, HV, d_v]")
    if HV != H and not ex:
        raise ValueError(f"{fn_name} takes H value heads; use decode_step_ex for num_v_heads != H")
    if HV % H != 0:
        raise ValueError("the number of value heads must be a multiple of the key heads")
    _check_state(S, (B, HV, dk, dv), dev)
    if o is None:
        o = torch.empty((B, HV, dv), dtype=q.dtype, device=dev)
    _check_tokens((o,), q.dtype, dev)
    if tuple(o.shape) != (B, HV, dv):
        raise ValueError(f"o must be {(B, HV, dv)}")
    with torch.cuda.device(dev):
        if ex:
            args = [_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w),
                    _ptr(S), _ptr(o), B, H, HV, dk, dv, _io(q.dtype)] + fuse(q, (B, HV, dv))
        else:
            args = [_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w),
                    _ptr(S), _ptr(o), B, H, dk, dv, _io(q.dtype)]
        st = getattr(lib(), fn_name)(*args, _stream(stream))
    if st != 0:
        raise Gdn2Error(st, fn_name)
    return o


def decode_step(q, k, v, log_alpha, b, w, S, *, o=None, stream=None):
    """One token per sequence: S [B,H,d_k,d_v] fp32 is updated in place; returns o [B,H,d_v]."""
    return _decode("gdn2_decode_step", q, k, v, log_alpha, b, w, S, o, stream)


def decode_step_ex(q, k, v, log_alpha, b, w, S, *, prep: bool = False, allow_neg_eigval: bool = False,
                   l2_eps: float = 1e-6, gate=None, norm_weight=None, norm_eps: float = 1e-5,
                   o=None, stream=None):
    """Decode step with value heads (v, w, gate [B,HV,d_v], S [B,HV,d_k,d_v]), the
    fused input prep and (gate, norm_weight [d_v]) the gated RMS-norm output
    epilogue."""
    fuse = lambda q_, shape: _fuse_args(q_, prep, allow_neg_eigval, l2_eps, gate, norm_weight,
                                        norm_eps, shape)
    return _decode("gdn2_decode_step_ex", q, k, v, log_alpha, b, w, S, o, stream, fuse, ex=True)


def chunk_fwd_qed(q, k, v, log_alpha, b, c, w, S0=None, *, qed_eps: float = 1e-6, o=None, S_T=None,
                  stream=None, want_state: bool = True):
    """Chunk forward with the second erase direction u_t (the part of q_t orthogonal to
    k_t, normalised) gated by c [B,T,H,d_k]; returns (o [B,T,H,d_v], S_T)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    _check_tokens((q, k, v, log_alpha, b, c, w), q.dtype, dev)
    for t in (k, log_alpha, b, c):
        if tuple(t.shape) != (B, T, H, dk):
            raise ValueError("q, k, log_alpha, b, c must be [B, T, H, d_k]")
    if tuple(w.shape) != (B, T, H, dv) or tuple(v.shape) != (B, T, H, dv):
        raise ValueError("v, w must be [B, T, H, d_v]")
    _check_state(S0, (B, H, dk, dv), dev)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=q.dtype, device=dev)
    if S_T is None and want_state:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    _check_tokens((o,), q.dtype, dev)
    _check_state(S_T, (B, H, dk, dv), dev)
    with torch.cuda.device(dev):
        st = lib().gdn2_chunk_fwd_qed(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(c), _ptr(w),
                                      _ptr(S0), _ptr(o), _ptr(S_T), B, T, H, dk, dv, _io(q.dtype),
                                      ctypes.c_float(float(qed_eps)), _stream(stream))
    if st != 0:
        raise Gdn2Error(st, "gdn2_chunk_fwd_qed")
    return o, S_T


def decode_step_qed(q, k, v, log_alpha, b, c, w, S, *, qed_eps: float = 1e-6, o=None, stream=None):
    """One token per sequence with the second erase direction; S [B,H,d_k,d_v] fp32
    is updated in place; returns o [B,H,d_v]."""
    B, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    _check_tokens((q, k, v, log_alpha, b, c, w), q.dtype, dev)
    for t in (k, log_alpha, b, c):
        if tuple(t.shape) != (B, H, dk):
            raise ValueError("q, k, log_alpha, b, c must be [B, H, d_k]")
    _check_state(S, (B, H, dk, dv), dev)
    if o is None:
        o = torch.empty((B, H, dv), dtype=q.dtype, device=dev)
    with torch.cuda.device(dev):
        st = lib().gdn2_decode_step_qed(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(c), _ptr(w),
                                        _ptr(S), _ptr(o), B, H, dk, dv, _io(q.dtype),
                                        ctypes.c_float(float(qed_eps)), _stream(stream))
    if st != 0:
        raise Gdn2Error(st, "gdn2_decode_step_qed")
    return o


def device_status(stream=None) -> int:
    """Synchronise the stream and read/clear the device status word."""
    return int(lib().gdn2_device_status(_stream(stream)))


def selftest_wait_timeout(limit_us: int = 1000, stream=None) -> int:
    return int(lib().gdn2_selftest_wait_timeout(int(limit_us), _stream(stream)))


def debug_bounds_site(stream=None):
    """Debug build: (buffer name, source line) of the first failed range check
    since the last read, or None; clears it.  Raises Gdn2Error in the release
    build (GDN2_ERR_UNSUPPORTED)."""
    buf, line = ctypes.c_int(-1), ctypes.c_int(0)
    st = lib().gdn2_debug_bounds_site(ctypes.byref(buf), ctypes.byref(line), _stream(stream))
    if st != 0:
        raise Gdn2Error(st, "gdn2_debug_bounds_site")
    return None if buf.value < 0 else (BOUNDS_BUFFERS[buf.value], line.value)


def testing_fail_launches(pass_: int, fail: int) -> None:
    """Fault injection for tests: after `pass_` more kernel launch sites, the
    next `fail` ones return GDN2_ERR_CUDA without launching; fail = 0 disarms."""
    st = lib().gdn2_testing_fail_launches(int(pass_), int(fail))
    if st != 0:
        raise Gdn2Error(st, "gdn2_testing_fail_launches")


def selftest_bounds(stream=None) -> int:
    """Debug build: GDN2_ERR_OUT_OF_BOUNDS when the range check works."""
    return int(lib().gdn2_selftest_bounds(_stream(stream)))
