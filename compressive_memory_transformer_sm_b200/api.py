"""ctypes binding of libinfini_attn (argument marshalling only).

Every function here has the name of the C entry point it calls and does no
arithmetic of its own: it reads shapes, data pointers and the current CUDA
stream from torch tensors and passes them on.  Importing this module loads
the in-tree shared library and raises ``ImportError`` when it has not been
built -- there is no CPU fallback.
"""

from __future__ import annotations

import ctypes
import os

import torch

from . import DELTA, F32, LINEAR  # noqa: F401

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "libinfini_attn.so")

INFINI_OK = 0
INFINI_ERR_INVALID_ARG = -1
INFINI_ERR_UNSUPPORTED = -2
INFINI_ERR_WORKSPACE = -3
INFINI_ERR_LAUNCH = -4
INFINI_ERR_TIMEOUT = -5
INFINI_ERR_DEVICE = -6
INFINI_ERR_SCRATCH_LIMIT = -7
NOALLOC_SCRATCH_BYTES = 32 << 20
FLAG_FORCE_SIMT = 0x1
FLAG_ATTN_SINGLE = 0x2
FLAG_ATTN_PAIRS = 0x4
FLAG_ATTN_SPLIT = 0x8

EXPORTED = (
    "infini_attn_forward", "infini_attn_segment_step", "infini_attn_forward_ex", "infini_attn_workspace_size",
    "infini_attn_error_string", "infini_attn_device_status", "infini_attn_selftest_timeout",
    "infini_attn_params_size", "infini_attn_path", "infini_attn_profile_enable", "infini_attn_profile_read",
    "infini_attn_launch_count", "infini_attn_forward_noalloc",
    "infini_attn_layer_forward", "infini_attn_layer_workspace_size", "infini_attn_decode_step",
    "infini_attn_workspace_size_ex", "infini_attn_gemm_bf16", "infini_attn_backward",
    "infini_attn_backward_workspace_size", "infini_attn_trim_workspace", "infini_attn_last_cuda_error",
)


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"libinfini_attn.so is not built ({_LIB_PATH}); run "
                          "`python -m compressive_memory_transformer_sm_b200.build`")
    return ctypes.CDLL(_LIB_PATH)


lib = _load()
_vp, _i, _l, _ll = ctypes.c_void_p, ctypes.c_int, ctypes.c_long, ctypes.c_longlong
lib.infini_attn_forward.argtypes = [_vp] * 7 + [_i, _i, _l, _i, _i, _i, _i, _vp]
lib.infini_attn_forward.restype = _i
lib.infini_attn_forward_noalloc.argtypes = [_vp] * 7 + [_i, _i, _l, _i, _i, _i, _i, _vp]
lib.infini_attn_forward_noalloc.restype = _i
lib.infini_attn_segment_step.argtypes = [_vp] * 7 + [_i, _i, _i, _i, _i, _i, _vp]
lib.infini_attn_segment_step.restype = _i
lib.infini_attn_workspace_size.argtypes = [_i, _i, _l, _i, _i, _i, _i]
lib.infini_attn_workspace_size.restype = ctypes.c_size_t
lib.infini_attn_error_string.argtypes = [_i]
lib.infini_attn_error_string.restype = ctypes.c_char_p
lib.infini_attn_device_status.argtypes = [_i]
lib.infini_attn_device_status.restype = _i
lib.infini_attn_selftest_timeout.argtypes = [ctypes.c_uint, _vp]
lib.infini_attn_selftest_timeout.restype = _i
lib.infini_attn_params_size.argtypes = []
lib.infini_attn_params_size.restype = ctypes.c_size_t
lib.infini_attn_path.argtypes = [_i, _i, _i, _i]
lib.infini_attn_path.restype = _i
lib.infini_attn_profile_enable.argtypes = [_i]
lib.infini_attn_profile_enable.restype = _i
lib.infini_attn_profile_read.argtypes = [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_ll), _i]
lib.infini_attn_profile_read.restype = _i
lib.infini_attn_launch_count.argtypes = []
lib.infini_attn_launch_count.restype = _ll
lib.infini_attn_last_cuda_error.argtypes = [ctypes.c_char_p, _i]
lib.infini_attn_last_cuda_error.restype = _i
lib.infini_attn_decode_step.argtypes = [_vp] * 9 + [_i] * 8 + [_vp]
lib.infini_attn_decode_step.restype = _i
lib.infini_attn_layer_forward.argtypes = [_vp] * 7 + [_i, _i, _l, _i, _i, _i, _vp, ctypes.c_size_t, _vp]
lib.infini_attn_layer_forward.restype = _i
lib.infini_attn_layer_workspace_size.argtypes = [_i, _i, _l, _i, _i, _i]
lib.infini_attn_layer_workspace_size.restype = ctypes.c_size_t
lib.infini_attn_gemm_bf16.argtypes = [_vp, _vp, _vp, _l, _i, _i, _vp]
lib.infini_attn_gemm_bf16.restype = _i

PHASE_UPDATE, PHASE_STATE, PHASE_ATTN, PHASE_PRE, PHASE_PROJ, PHASE_BWD, PHASE_BWD_TC, PHASE_BWD_MEM_TC = range(8)
PHASES = 8


class InfiniAttnParams(ctypes.Structure):
    """Mirror of ``infini_attn_params`` (include/infini_attn.h)."""

    _fields_ = [
        ("q", _vp), ("k", _vp), ("v", _vp), ("beta", _vp), ("M", _vp), ("z", _vp), ("out", _vp),
        ("B", _i), ("H", _i), ("L", _ll), ("N", _i), ("dk", _i), ("dv", _i), ("mode", _i),
        ("scale", ctypes.c_float),
        ("q_stride", _ll * 3), ("k_stride", _ll * 3), ("v_stride", _ll * 3), ("o_stride", _ll * 3),
        ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t), ("flags", _i), ("stream", _vp),
        ("rope_base", ctypes.c_double), ("rope_offset", _ll),
    ]


lib.infini_attn_forward_ex.argtypes = [ctypes.POINTER(InfiniAttnParams)]
lib.infini_attn_forward_ex.restype = _i
lib.infini_attn_workspace_size_ex.argtypes = [ctypes.POINTER(InfiniAttnParams)]
lib.infini_attn_workspace_size_ex.restype = ctypes.c_size_t


class InfiniAttnBwdParams(ctypes.Structure):
    """Mirror of ``infini_attn_bwd_params`` (include/infini_attn.h)."""

    _fields_ = [
        ("q", _vp), ("k", _vp), ("v", _vp), ("beta", _vp), ("M0", _vp), ("z0", _vp), ("d_out", _vp),
        ("dM_S", _vp), ("dz_S", _vp), ("dq", _vp), ("dk", _vp), ("dv", _vp), ("dbeta", _vp), ("dM0", _vp),
        ("dz0", _vp), ("B", _i), ("H", _i), ("L", _ll), ("N", _i), ("d_k", _i), ("d_v", _i), ("mode", _i),
        ("scale", ctypes.c_float), ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t), ("stream", _vp),
        ("flags", _i),
    ]


lib.infini_attn_backward.argtypes = [ctypes.POINTER(InfiniAttnBwdParams)]
lib.infini_attn_backward.restype = _i
lib.infini_attn_backward_workspace_size.argtypes = [ctypes.POINTER(InfiniAttnBwdParams)]
lib.infini_attn_backward_workspace_size.restype = ctypes.c_size_t
lib.infini_attn_trim_workspace.argtypes = []
lib.infini_attn_trim_workspace.restype = _i


class InfiniAttnError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        detail = ""
        if code == INFINI_ERR_LAUNCH:
            err, name = infini_attn_last_cuda_error()
            detail = f" [{name} ({err})]" if err else ""
        super().__init__(f"{where}: {infini_attn_error_string(code)} ({code}){detail}")


def infini_attn_last_cuda_error():
    """(cudaError_t value, its name) behind the most recent INFINI_ERR_LAUNCH of this library; (0, ...) if none."""
    buf = ctypes.create_string_buffer(64)
    err = int(lib.infini_attn_last_cuda_error(buf, len(buf)))
    return err, buf.value.decode()


def infini_attn_error_string(code: int) -> str:
    return lib.infini_attn_error_string(int(code)).decode()


def infini_attn_trim_workspace() -> None:
    """Return the unused device memory of the library's own workspace pool (current context) to the driver."""
    rc = lib.infini_attn_trim_workspace()
    if rc != 0:
        raise InfiniAttnError(rc, "infini_attn_trim_workspace")


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _mode(mode: int, t: torch.Tensor) -> int:
    return int(mode) | (F32 if t.dtype == torch.float32 else 0)


def _args(where: str, shapes: dict, contiguous: bool = True):
    """Marshalling checks before a pointer leaves Python: every tensor on a CUDA device, with the
    expected number of dimensions, contiguous unless the call takes strides; raises ValueError."""
    for name, (t, ndim) in shapes.items():
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{where}: {name} must be a torch.Tensor")
        if t.dim() != ndim:
            raise ValueError(f"{where}: {name} must have {ndim} dimensions, got shape {tuple(t.shape)}")
        if not t.is_cuda:
            raise ValueError(f"{where}: {name} must be on a CUDA device, got {t.device}")
        if contiguous and not t.is_contiguous():
            raise ValueError(f"{where}: {name} must be contiguous (use infini_attn_forward_ex for strided views)")


def _same(where: str, what: str, *vals):
    if len(set(vals)) != 1:
        raise ValueError(f"{where}: {what} disagree: {vals}")


def _check(rc: int, where: str, raise_on_error: bool):
    if rc != INFINI_OK and raise_on_error:
        raise InfiniAttnError(rc, where)
    return rc


def infini_attn_forward(q, k, v, beta, M, z, out, N: int, mode: int = LINEAR, stream=None, raise_on_error=True):
    """q, k [B,H,L,dk], v, out [B,H,L,dv] (bf16 or fp32, contiguous); beta [H]; M [B,H,dk,dv]; z [B,H,dk]."""
    _args("infini_attn_forward", dict(q=(q, 4), k=(k, 4), v=(v, 4), out=(out, 4), beta=(beta, 1), M=(M, 4),
                                      z=(z, 3)))
    B, H, L, dk = q.shape
    dv = v.shape[3]
    _same("infini_attn_forward", "q / k / v / out (B, H, L)", tuple(q.shape[:3]), tuple(k.shape[:3]),
          tuple(v.shape[:3]), tuple(out.shape[:3]))
    rc = lib.infini_attn_forward(q.data_ptr(), k.data_ptr(), v.data_ptr(), beta.data_ptr(), M.data_ptr(),
                                 z.data_ptr(), out.data_ptr(), B, H, L, int(N), dk, dv, _mode(mode, q),
                                 _stream(stream))
    return _check(rc, "infini_attn_forward", raise_on_error)


def infini_attn_forward_noalloc(q, k, v, beta, M, z, out, N: int, mode: int = LINEAR, stream=None,
                                raise_on_error=True):
    """infini_attn_forward for callers that must not allocate device memory during the call.

    The workspace comes from the library's fixed 32 MiB device buffer instead of
    cudaMallocAsync; shapes needing more are refused (INFINI_ERR_SCRATCH_LIMIT).  Calls that
    overlap on the GPU share that buffer and race, so keep them on one stream.
    """
    _args("infini_attn_forward_noalloc", dict(q=(q, 4), k=(k, 4), v=(v, 4), out=(out, 4), beta=(beta, 1),
                                              M=(M, 4), z=(z, 3)))
    B, H, L, dk = q.shape
    dv = v.shape[3]
    _same("infini_attn_forward_noalloc", "q / k / v / out (B, H, L)", tuple(q.shape[:3]), tuple(k.shape[:3]),
          tuple(v.shape[:3]), tuple(out.shape[:3]))
    rc = lib.infini_attn_forward_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), beta.data_ptr(), M.data_ptr(),
                                         z.data_ptr(), out.data_ptr(), B, H, L, int(N), dk, dv, _mode(mode, q),
                                         _stream(stream))
    return _check(rc, "infini_attn_forward_noalloc", raise_on_error)


def infini_attn_segment_step(q, k, v, beta, M, z, out, mode: int = LINEAR, stream=None, raise_on_error=True):
    """One segment of n tokens per (b, h): q, k [B,H,n,dk], v, out [B,H,n,dv]."""
    _args("infini_attn_segment_step", dict(q=(q, 4), k=(k, 4), v=(v, 4), out=(out, 4), beta=(beta, 1),
                                           M=(M, 4), z=(z, 3)))
    B, H, n, dk = q.shape
    dv = v.shape[3]
    _same("infini_attn_segment_step", "q / k / v / out (B, H, n)", tuple(q.shape[:3]), tuple(k.shape[:3]),
          tuple(v.shape[:3]), tuple(out.shape[:3]))
    rc = lib.infini_attn_segment_step(q.data_ptr(), k.data_ptr(), v.data_ptr(), beta.data_ptr(), M.data_ptr(),
                                      z.data_ptr(), out.data_ptr(), B, H, n, dk, dv, _mode(mode, q),
                                      _stream(stream))
    return _check(rc, "infini_attn_segment_step", raise_on_error)


def infini_attn_decode_step(q_t, k_t, v_t, k_cache, v_cache, beta, M, z, out, pos: int, mode: int = LINEAR,
                            fold: bool = False, stream=None, raise_on_error=True):
    """One token per (b, h) at position ``pos`` of the current segment: q_t, k_t [B,H,dk], v_t, out [B,H,dv];
    k_cache [B,H,N,dk], v_cache [B,H,N,dv] (same dtype, bf16 or fp32); folds the segment into M, z when
    pos == N - 1 or ``fold``."""
    _args("infini_attn_decode_step", dict(q_t=(q_t, 3), k_t=(k_t, 3), v_t=(v_t, 3), k_cache=(k_cache, 4),
                                          v_cache=(v_cache, 4), out=(out, 3), beta=(beta, 1), M=(M, 4), z=(z, 3)))
    B, H, dk = q_t.shape
    dv = v_t.shape[2]
    N = k_cache.shape[2]
    _same("infini_attn_decode_step", "token and cache (B, H)", tuple(q_t.shape[:2]), tuple(k_t.shape[:2]),
          tuple(v_t.shape[:2]), tuple(out.shape[:2]), tuple(k_cache.shape[:2]), tuple(v_cache.shape[:2]))
    _same("infini_attn_decode_step", "cache lengths", k_cache.shape[2], v_cache.shape[2])
    rc = lib.infini_attn_decode_step(q_t.data_ptr(), k_t.data_ptr(), v_t.data_ptr(), k_cache.data_ptr(),
                                     v_cache.data_ptr(), beta.data_ptr(), M.data_ptr(), z.data_ptr(), out.data_ptr(),
                                     B, H, N, int(pos), dk, dv, _mode(mode, q_t), int(bool(fold)), _stream(stream))
    return _check(rc, "infini_attn_decode_step", raise_on_error)


def infini_attn_layer_forward(x, w_qkv, w_o, beta, M, z, y, H: int, N: int, mode: int = LINEAR, workspace=None,
                              stream=None, raise_on_error=True):
    """Full layer: x [B,L,D] bf16; w_qkv [D, 3*H*128] (Q | K | V column blocks, head-major); w_o [H*128, D];
    y [B,L,D] bf16 (written); beta [H]; M [B,H,128,128]; z [B,H,128].  workspace: optional uint8 device
    tensor of at least infini_attn_layer_workspace_size(...) bytes."""
    _args("infini_attn_layer_forward", dict(x=(x, 3), w_qkv=(w_qkv, 2), w_o=(w_o, 2), y=(y, 3), beta=(beta, 1),
                                            M=(M, 4), z=(z, 3)))
    B, L, D = x.shape
    _same("infini_attn_layer_forward", "x / y shapes", tuple(x.shape), tuple(y.shape))
    if tuple(w_qkv.shape) != (D, 3 * int(H) * 128) or tuple(w_o.shape) != (int(H) * 128, D):
        raise ValueError(f"infini_attn_layer_forward: w_qkv must be [{D}, {3 * int(H) * 128}] and w_o "
                         f"[{int(H) * 128}, {D}], got {tuple(w_qkv.shape)} and {tuple(w_o.shape)}")
    ws, wsb = (workspace.data_ptr(), workspace.numel() * workspace.element_size()) if workspace is not None else (None, 0)
    rc = lib.infini_attn_layer_forward(x.data_ptr(), w_qkv.data_ptr(), w_o.data_ptr(), beta.data_ptr(), M.data_ptr(),
                                       z.data_ptr(), y.data_ptr(), B, int(H), L, int(N), D, int(mode), ws, wsb,
                                       _stream(stream))
    return _check(rc, "infini_attn_layer_forward", raise_on_error)


def infini_attn_gemm_bf16(a, b, c, stream=None, raise_on_error=True):
    """c[M, N] = a[M, K] @ b[K, N]: contiguous bf16 device matrices, fp32 accumulation (the layer's projection)."""
    _args("infini_attn_gemm_bf16", dict(a=(a, 2), b=(b, 2), c=(c, 2)))
    M, K = a.shape
    N = b.shape[1]
    if b.shape[0] != K or tuple(c.shape) != (M, N):
        raise ValueError(f"infini_attn_gemm_bf16: shapes {tuple(a.shape)} @ {tuple(b.shape)} -> {tuple(c.shape)}")
    for name, t in (("a", a), ("b", b), ("c", c)):
        if t.dtype != torch.bfloat16:
            raise ValueError(f"infini_attn_gemm_bf16: {name} must be bfloat16")
    rc = lib.infini_attn_gemm_bf16(a.data_ptr(), b.data_ptr(), c.data_ptr(), M, N, K, _stream(stream))
    return _check(rc, "infini_attn_gemm_bf16", raise_on_error)


def infini_attn_layer_workspace_size(B, H, L, N, d_model, mode=LINEAR) -> int:
    return int(lib.infini_attn_layer_workspace_size(B, H, L, N, d_model, mode))


def _bhl_strides(t: torch.Tensor):
    """Element strides of the (B, H, L) dimensions of a [B, H, L, d] view with d contiguous."""
    if t.stride(3) != 1:
        raise ValueError("the last dimension must be contiguous")
    return (t.stride(0), t.stride(1), t.stride(2))


def infini_attn_forward_ex(q, k, v, beta, M, z, out, N: int, mode: int = LINEAR, scale: float = 0.0,
                           workspace=None, flags: int = 0, stream=None, raise_on_error=True, rope_base: float = 0.0,
                           rope_offset: int = 0):
    """Extended call: [B,H,L,d] views with any (B, H, L) strides, explicit scale, caller workspace, flags, and
    rotary position embeddings on the local attention only (``rope_base`` > 0, token t at position
    ``rope_offset + t``)."""
    _args("infini_attn_forward_ex", dict(q=(q, 4), k=(k, 4), v=(v, 4), out=(out, 4)), contiguous=False)
    _args("infini_attn_forward_ex", dict(beta=(beta, 1), M=(M, 4), z=(z, 3)))
    B, H, L, dk = q.shape
    dv = v.shape[3]
    p = InfiniAttnParams()
    p.q, p.k, p.v, p.beta = q.data_ptr(), k.data_ptr(), v.data_ptr(), beta.data_ptr()
    p.M, p.z, p.out = M.data_ptr(), z.data_ptr(), out.data_ptr()
    p.B, p.H, p.L, p.N, p.dk, p.dv = B, H, L, int(N), dk, dv
    p.mode = _mode(mode, q)
    p.scale = float(scale)
    for name, t in (("q_stride", q), ("k_stride", k), ("v_stride", v), ("o_stride", out)):
        getattr(p, name)[:] = _bhl_strides(t)
    if workspace is not None:
        p.workspace = workspace.data_ptr()
        p.workspace_bytes = workspace.numel() * workspace.element_size()
    p.flags = int(flags)
    p.stream = _stream(stream)
    p.rope_base = float(rope_base)
    p.rope_offset = int(rope_offset)
    rc = lib.infini_attn_forward_ex(ctypes.byref(p))
    return _check(rc, "infini_attn_forward_ex", raise_on_error)


def _ptr(t):
    return None if t is None else t.data_ptr()


def infini_attn_backward(q, k, v, beta, d_out, N: int, mode: int = LINEAR, M0=None, z0=None, dM_S=None, dz_S=None,
                         want_state_grad: bool = True, scale: float = 0.0, workspace=None, flags: int = 0,
                         stream=None, raise_on_error=True):
    """Gradients through the forward: returns (dq, dk, dv, dbeta, dM0, dz0) as new device tensors
    (dM0, dz0 are None unless ``want_state_grad``).  q, k [B,H,L,dk], v, d_out [B,H,L,dv] contiguous,
    one dtype (bf16 or fp32); beta [H]; M0, dM_S [B,H,dk,dv], z0, dz_S [B,H,dk] fp32 or None."""
    _args("infini_attn_backward", dict(q=(q, 4), k=(k, 4), v=(v, 4), d_out=(d_out, 4), beta=(beta, 1)))
    for name, t, nd in (("M0", M0, 4), ("z0", z0, 3), ("dM_S", dM_S, 4), ("dz_S", dz_S, 3)):
        if t is not None:
            _args("infini_attn_backward", {name: (t, nd)})
    B, H, L, dk = q.shape
    dv = v.shape[3]
    _same("infini_attn_backward", "q / k / v / d_out (B, H, L)", tuple(q.shape[:3]), tuple(k.shape[:3]),
          tuple(v.shape[:3]), tuple(d_out.shape[:3]))
    dq, dk_, dv_ = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dbeta = torch.empty(H, dtype=torch.float32, device=q.device)
    dM0 = torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device) if want_state_grad else None
    dz0 = torch.empty(B, H, dk, dtype=torch.float32, device=q.device) if want_state_grad else None
    p = InfiniAttnBwdParams()
    p.q, p.k, p.v, p.beta, p.d_out = q.data_ptr(), k.data_ptr(), v.data_ptr(), beta.data_ptr(), d_out.data_ptr()
    p.M0, p.z0, p.dM_S, p.dz_S = _ptr(M0), _ptr(z0), _ptr(dM_S), _ptr(dz_S)
    p.dq, p.dk, p.dv, p.dbeta, p.dM0, p.dz0 = dq.data_ptr(), dk_.data_ptr(), dv_.data_ptr(), dbeta.data_ptr(), \
        _ptr(dM0), _ptr(dz0)
    p.B, p.H, p.L, p.N, p.d_k, p.d_v = B, H, L, int(N), dk, dv
    p.mode = _mode(mode, q)
    p.scale = float(scale)
    if workspace is not None:
        p.workspace = workspace.data_ptr()
        p.workspace_bytes = workspace.numel() * workspace.element_size()
    p.stream = _stream(stream)
    p.flags = int(flags)
    rc = lib.infini_attn_backward(ctypes.byref(p))
    _check(rc, "infini_attn_backward", raise_on_error)
    return dq, dk_, dv_, dbeta, dM0, dz0


def infini_attn_backward_workspace_size(B, H, L, N, dk, dv, mode=LINEAR, flags: int = 0) -> int:
    p = InfiniAttnBwdParams()
    p.B, p.H, p.L, p.N, p.d_k, p.d_v, p.mode = int(B), int(H), int(L), int(N), int(dk), int(dv), int(mode)
    p.flags = int(flags)
    return int(lib.infini_attn_backward_workspace_size(ctypes.byref(p)))


def infini_attn_workspace_size(B, H, L, N, dk, dv, mode=LINEAR) -> int:
    return int(lib.infini_attn_workspace_size(B, H, L, N, dk, dv, mode))


def infini_attn_workspace_size_ex(B, H, L, N, dk, dv, mode=LINEAR, rope_base: float = 0.0) -> int:
    """Workspace of infini_attn_forward_ex for this shape, including the rotated q, k when rope_base > 0."""
    p = InfiniAttnParams()
    p.B, p.H, p.L, p.N, p.dk, p.dv, p.mode = int(B), int(H), int(L), int(N), int(dk), int(dv), int(mode)
    p.rope_base = float(rope_base)
    return int(lib.infini_attn_workspace_size_ex(ctypes.byref(p)))


def infini_attn_device_status(reset: bool = False) -> int:
    return int(lib.infini_attn_device_status(1 if reset else 0))


def infini_attn_selftest_timeout(limit_us: int, stream=None) -> int:
    return int(lib.infini_attn_selftest_timeout(int(limit_us), _stream(stream)))


def infini_attn_path(dk: int, dv: int, mode: int, flags: int = 0) -> int:
    return int(lib.infini_attn_path(dk, dv, mode, flags))


def infini_attn_profile_enable(phase_mask: int) -> int:
    return int(lib.infini_attn_profile_enable(int(phase_mask)))


def infini_attn_profile_read(reset: bool = True):
    """Returns ([ms per phase], [timed launches per phase]) for the phases PHASE_UPDATE ..
    PHASE_BWD_MEM_TC (memory update, state, attention, position-embedding pre-pass, projections,
    backward on CUDA cores, local attention's backward and memory branch's backward on the tensor
    cores)."""
    ms = (ctypes.c_double * PHASES)()
    n = (_ll * PHASES)()
    rc = lib.infini_attn_profile_read(ms, n, 1 if reset else 0)
    if rc != INFINI_OK:
        raise InfiniAttnError(rc, "infini_attn_profile_read")
    return list(ms), list(n)


def infini_attn_launch_count() -> int:
    return int(lib.infini_attn_launch_count())


def forward_host(q, k, v, beta, M, z, N: int, mode: int = LINEAR, device="cuda", out=None, stream=None):
    """End-to-end call with HOST tensors: copy inputs to the device, run, copy the output and state back.

    q, k, v, beta, M, z are CPU tensors (pinned for asynchronous copies); returns (out, M, z) on the host.
    """
    dev = torch.device(device)
    s = torch.cuda.current_stream(dev) if stream is None else stream
    with torch.cuda.stream(s):
        qd, kd, vd = (t.to(dev, non_blocking=True) for t in (q, k, v))
        bd, Md, zd = (t.to(dev, non_blocking=True) for t in (beta, M, z))
        od = torch.empty(q.shape[:3] + (v.shape[3],), dtype=q.dtype, device=dev)
        infini_attn_forward(qd, kd, vd, bd, Md, zd, od, N, mode, stream=s)
        if out is None:
            out = torch.empty(od.shape, dtype=od.dtype, pin_memory=True)
        out.copy_(od, non_blocking=True)
        M.copy_(Md, non_blocking=True)
        z.copy_(zd, non_blocking=True)
    return out, M, z
