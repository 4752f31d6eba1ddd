"""The C-ABI library loads, exports what include/infini_attn.h declares, and validates on the host.

No test here launches a kernel: argument checks run before any CUDA call,
and on a machine without a GPU a well-formed call reports INFINI_ERR_DEVICE.
"""

import ctypes
import os
import re

import pytest
import torch

from compressive_memory_transformer_sm_b200 import DELTA, F32, LINEAR, api

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "infini_attn.h")


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"INFINI_API\s+[\w\s\*]+?\b(infini_attn_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("infini_attn_forward", "infini_attn_segment_step", "infini_attn_forward_ex",
                     "infini_attn_workspace_size", "infini_attn_error_string"):
        assert required in names


def test_library_exports_every_declared_symbol():
    for name in declared_functions():
        assert hasattr(api.lib, name), name
        assert ctypes.cast(getattr(api.lib, name), ctypes.c_void_p).value
    assert set(api.EXPORTED) == set(declared_functions())


def test_params_struct_layout_matches():
    assert api.lib.infini_attn_params_size() == ctypes.sizeof(api.InfiniAttnParams)


def test_error_strings():
    for code in (0, -1, -2, -3, -4, -5, -6, -99, 7):
        s = api.infini_attn_error_string(code)
        assert isinstance(s, str) and s
    assert api.infini_attn_error_string(-99) == "unknown error code"


def test_last_cuda_error_query():
    # code and name agree (0 is cudaSuccess); a NULL buffer or a zero length
    # is accepted and a short buffer is truncated, NUL-terminated
    err, name = api.infini_attn_last_cuda_error()
    assert isinstance(err, int) and name and (err == 0) == (name == "cudaSuccess")
    assert api.lib.infini_attn_last_cuda_error(None, 0) == err
    buf = ctypes.create_string_buffer(4)
    assert api.lib.infini_attn_last_cuda_error(buf, len(buf)) == err and buf.value == name[:3].encode()


def test_path_selection():
    assert api.infini_attn_path(128, 128, LINEAR, 0) == 1
    assert api.infini_attn_path(128, 128, DELTA, 0) == 1
    assert api.infini_attn_path(128, 128, LINEAR | F32, 0) == 0
    assert api.infini_attn_path(128, 128, LINEAR, api.FLAG_FORCE_SIMT) == 0
    assert api.infini_attn_path(64, 128, LINEAR, 0) == 0
    assert api.infini_attn_path(16, 16, DELTA | F32, 0) == 0
    assert api.infini_attn_path(129, 128, LINEAR, 0) == api.INFINI_ERR_UNSUPPORTED
    assert api.infini_attn_path(128, 128, 0x4, 0) == api.INFINI_ERR_UNSUPPORTED
    assert api.infini_attn_path(0, 128, LINEAR, 0) == api.INFINI_ERR_INVALID_ARG


def test_workspace_size_is_deterministic_and_bounded():
    a = api.infini_attn_workspace_size(1, 8, 32768, 2048, 128, 128, LINEAR)
    assert a == api.infini_attn_workspace_size(1, 8, 32768, 2048, 128, 128, LINEAR) and a > 0
    # snapshots alone: 16 segments x 8 heads x (128*128 fp32 + 128 fp32)
    assert a >= 16 * 8 * (128 * 128 * 4 + 128 * 4)
    assert api.infini_attn_workspace_size(0, 8, 32768, 2048, 128, 128, LINEAR) == 0
    assert api.infini_attn_workspace_size(1, 8, 0, 2048, 128, 128, LINEAR) == 0
    assert api.infini_attn_workspace_size(1, 8, 32768, 2048, 256, 128, LINEAR) == 0
    # delta reuses one segment of partials: never more than linear for the same shape
    assert api.infini_attn_workspace_size(1, 8, 32768, 2048, 128, 128, DELTA) <= a


def _call(**over):
    args = dict(q=1 << 20, k=2 << 20, v=3 << 20, beta=4 << 20, M=5 << 20, z=6 << 20, out=7 << 20,
                B=1, H=2, L=64, N=16, dk=16, dv=16, mode=LINEAR | F32, stream=None)
    args.update(over)
    return api.lib.infini_attn_forward(args["q"], args["k"], args["v"], args["beta"], args["M"], args["z"],
                                       args["out"], args["B"], args["H"], args["L"], args["N"], args["dk"],
                                       args["dv"], args["mode"], args["stream"])


@pytest.mark.parametrize("over,code", [
    (dict(q=None), -1), (dict(k=None), -1), (dict(v=None), -1), (dict(beta=None), -1), (dict(M=None), -1),
    (dict(z=None), -1), (dict(out=None), -1), (dict(B=0), -1), (dict(H=-1), -1), (dict(L=0), -1),
    (dict(N=0), -1), (dict(dk=0), -1), (dict(dk=129), -2), (dict(dv=200), -2), (dict(mode=0x4), -2),
    (dict(out=1 << 20), -1),            # out aliases q
    (dict(z=5 << 20), -1),              # z aliases M
])
def test_invalid_arguments_rejected_on_host(over, code):
    assert _call(**over) == code


def test_segment_step_rejects_empty_segment():
    rc = api.lib.infini_attn_segment_step(1 << 20, 2 << 20, 3 << 20, 4 << 20, 5 << 20, 6 << 20, 7 << 20,
                                          1, 2, 0, 16, 16, LINEAR, None)
    assert rc == api.INFINI_ERR_INVALID_ARG


def test_forward_ex_rejects_null_and_small_workspace():
    assert api.lib.infini_attn_forward_ex(None) == api.INFINI_ERR_INVALID_ARG
    p = api.InfiniAttnParams()
    p.q, p.k, p.v, p.beta, p.M, p.z, p.out = (i << 20 for i in range(1, 8))
    p.B, p.H, p.L, p.N, p.dk, p.dv, p.mode = 1, 2, 64, 16, 16, 16, LINEAR | F32
    p.workspace = 1 << 30
    p.workspace_bytes = 16
    assert api.lib.infini_attn_forward_ex(ctypes.byref(p)) == api.INFINI_ERR_WORKSPACE
    p.workspace_bytes = 1 << 30
    p.workspace = (1 << 30) + 8  # misaligned
    assert api.lib.infini_attn_forward_ex(ctypes.byref(p)) == api.INFINI_ERR_WORKSPACE


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU answer")
def test_wellformed_call_without_gpu_reports_device():
    assert _call() == api.INFINI_ERR_DEVICE


# ---------------------------------------------------------------- full layer
def _layer(**over):
    a = dict(x=1 << 20, w_qkv=2 << 20, w_o=3 << 20, beta=4 << 20, M=5 << 20, z=6 << 20, y=7 << 20,
             B=1, H=2, L=256, N=128, D=64, mode=LINEAR, ws=None, wsb=0)
    a.update(over)
    return api.lib.infini_attn_layer_forward(a["x"], a["w_qkv"], a["w_o"], a["beta"], a["M"], a["z"], a["y"],
                                             a["B"], a["H"], a["L"], a["N"], a["D"], a["mode"], a["ws"], a["wsb"],
                                             None)


@pytest.mark.parametrize("over,code", [
    (dict(x=None), -1), (dict(w_qkv=None), -1), (dict(w_o=None), -1), (dict(y=None), -1), (dict(M=None), -1),
    (dict(B=0), -1), (dict(D=0), -1), (dict(N=0), -1),
    (dict(mode=LINEAR | F32), -2),       # the layer is bf16 only
    (dict(y=(1 << 20) + 64), -1),        # y aliases x
    (dict(ws=1 << 30, wsb=16), -3),      # workspace too small
])
def test_layer_invalid_arguments_rejected_on_host(over, code):
    assert _layer(**over) == code


def test_layer_workspace_size():
    s = api.infini_attn_layer_workspace_size(1, 8, 32768, 2048, 1024, LINEAR)
    # Q, K, V and the attention output in bf16, plus the attention workspace
    assert s >= 32768 * (3 + 1) * 8 * 128 * 2 + api.infini_attn_workspace_size(1, 8, 32768, 2048, 128, 128, LINEAR)
    assert api.infini_attn_layer_workspace_size(1, 8, 32768, 2048, 0, LINEAR) == 0
    assert api.infini_attn_layer_workspace_size(1, 8, 32768, 2048, 1024, LINEAR | F32) == 0


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU answer")
def test_layer_wellformed_call_without_gpu_reports_device():
    assert _layer() == api.INFINI_ERR_DEVICE


# ---------------------------------------------------------------- streaming decode
def _decode(**over):
    a = dict(q=1 << 20, k=2 << 20, v=3 << 20, kc=4 << 20, vc=5 << 20, beta=6 << 20, M=7 << 20, z=8 << 20,
             out=9 << 20, B=1, H=2, N=64, pos=0, dk=128, dv=128, mode=LINEAR, fold=0)
    a.update(over)
    return api.lib.infini_attn_decode_step(a["q"], a["k"], a["v"], a["kc"], a["vc"], a["beta"], a["M"], a["z"],
                                           a["out"], a["B"], a["H"], a["N"], a["pos"], a["dk"], a["dv"], a["mode"],
                                           a["fold"], None)


@pytest.mark.parametrize("over,code", [
    (dict(q=None), -1), (dict(kc=None), -1), (dict(out=None), -1), (dict(B=0), -1), (dict(N=0), -1),
    (dict(pos=-1), -1), (dict(pos=64), -1), (dict(dk=129), -2), (dict(mode=0x4), -2),
])
def test_decode_invalid_arguments_rejected_on_host(over, code):
    assert _decode(**over) == code


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU answer")
def test_decode_wellformed_call_without_gpu_reports_device():
    assert _decode() == api.INFINI_ERR_DEVICE


# ---------------------------------------------------------------- Python marshalling checks
def test_binding_rejects_host_and_strided_tensors():
    q = torch.zeros(1, 2, 8, 16)
    with pytest.raises(ValueError, match="CUDA device"):
        api.infini_attn_forward(q, q, q, torch.zeros(2), torch.zeros(1, 2, 16, 16), torch.zeros(1, 2, 16), q, 4)
    with pytest.raises(ValueError, match="dimensions"):
        api.infini_attn_segment_step(q[0], q, q, torch.zeros(2), torch.zeros(1, 2, 16, 16), torch.zeros(1, 2, 16), q)
    with pytest.raises(ValueError):
        api.infini_attn_layer_forward(torch.zeros(1, 8, 64), torch.zeros(64, 3 * 128), torch.zeros(128, 64),
                                      torch.zeros(1), torch.zeros(1, 1, 128, 128), torch.zeros(1, 1, 128),
                                      torch.zeros(1, 8, 64), 1, 4)


def _call_ex(**over):
    p = api.InfiniAttnParams()
    vals = dict(q=1 << 20, k=2 << 20, v=3 << 20, beta=4 << 20, M=5 << 20, z=6 << 20, out=7 << 20,
                B=1, H=2, L=64, N=16, dk=16, dv=16, mode=LINEAR | F32, rope_base=10000.0, rope_offset=0)
    vals.update(over)
    for key, val in vals.items():
        setattr(p, key, val)
    return api.lib.infini_attn_forward_ex(ctypes.byref(p))


def test_rope_arguments_are_validated_before_any_cuda_call():
    assert _call_ex(rope_base=-1.0) == api.INFINI_ERR_INVALID_ARG
    assert _call_ex(rope_base=float("nan")) == api.INFINI_ERR_INVALID_ARG
    assert _call_ex(rope_base=float("inf")) == api.INFINI_ERR_INVALID_ARG
    assert _call_ex(dk=15) == api.INFINI_ERR_UNSUPPORTED  # pairs need an even head size
    # a valid call reaches the device check (no GPU here) or runs
    assert _call_ex() in (api.INFINI_ERR_DEVICE, api.INFINI_OK) or torch.cuda.is_available()


def test_workspace_size_ex_counts_the_rotated_copies():
    base = api.infini_attn_workspace_size(1, 8, 32768, 2048, 128, 128, LINEAR)
    assert api.infini_attn_workspace_size_ex(1, 8, 32768, 2048, 128, 128, LINEAR) == base
    with_rope = api.infini_attn_workspace_size_ex(1, 8, 32768, 2048, 128, 128, LINEAR, rope_base=10000.0)
    assert with_rope >= base + 2 * 8 * 32768 * 128 * 2  # rotated q and k in bf16
    assert api.infini_attn_workspace_size_ex(1, 8, 32768, 2048, 127, 128, LINEAR, rope_base=10000.0) == 0
    assert api.infini_attn_workspace_size_ex(1, 8, 32768, 2048, 128, 128, LINEAR, rope_base=-5.0) == 0
