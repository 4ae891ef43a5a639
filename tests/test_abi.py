"""CPU tests of the C ABI: the library loads, exports every declared symbol, and
rejects bad arguments synchronously without touching a GPU."""
import ctypes
import os
import subprocess

import pytest
import torch

import exact_tiled_attention_34_b200 as fa

OK, INVALID, UNSUPPORTED, ALIGN, WORKSPACE, CUDA = 0, 1, 2, 3, 4, 5


@pytest.fixture(scope="module")
def L():
    from exact_tiled_attention_34_b200 import build
    build.build()
    return fa.lib()


def test_exports_every_declared_symbol(L):
    names = fa.exported_names()
    assert {"fa_fwd", "fa_bwd", "fa_fwd_blocksparse", "fa_bwd_blocksparse", "fa_bwd_workspace_bytes",
            "fa_status_string", "fa_device_status", "fa_version", "fa_bwd_preprocess", "fa_bwd_dkdv",
            "fa_bwd_dq", "fa_bwd_noalloc", "fa_debug_wait_timeout",
            "fa_debug_stall_producer", "fa_fwd_dropout", "fa_bwd_dropout", "fa_merge_partial",
            "fa_accumulate_bf16", "fa_to_bf16", "fa_bwd_fused_workspace_bytes", "fa_bwd_fused", "fa_bwd_fused_ex",
            "fa_bwd_fused_preprocess", "fa_bwd_fused_main", "fa_bwd_fused_dq", "fa_fwd_merge", "fa_bwd_fused_main_f32",
            "fa_accumulate_f32"} <= set(names)
    out = subprocess.run(["nm", "-D", "--defined-only", fa.lib_path()], capture_output=True, text=True,
                         check=True).stdout
    defined = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [n for n in names if n not in defined]
    assert not missing, missing
    for n in names:
        assert getattr(L, n) is not None


def test_status_strings(L):
    for code, name in fa.STATUS.items():
        assert L.fa_status_string(code).decode() == name
    assert L.fa_status_string(99).decode() == "FA_ERR_UNKNOWN"
    assert L.fa_version() >= 100


A = 1 << 20  # fake, 16-byte aligned "device" addresses: never dereferenced by these checks

# A call with valid arguments and the fake addresses would launch a kernel on them when
# a GPU is present, so those calls are made only on a machine without one (where they
# stop at the first CUDA call and return FA_ERR_CUDA).
NO_GPU = not torch.cuda.is_available()


def _fwd(L, q=A, k=A, v=A, o=A, lse=A, B=1, H=1, N=128, d=64, causal=0, scale=0.125):
    return L.fa_fwd(q, k, v, o, lse, B, H, N, d, causal, scale, None)


def test_fwd_argument_checks(L):
    assert _fwd(L, q=None) == INVALID
    assert _fwd(L, lse=None) == INVALID
    assert _fwd(L, k=A + 8) == ALIGN
    assert _fwd(L, o=A + 2) == ALIGN
    assert _fwd(L, B=0) == INVALID
    assert _fwd(L, H=-1) == INVALID
    assert _fwd(L, N=0) == INVALID
    assert _fwd(L, d=32) == UNSUPPORTED
    if NO_GPU:
        assert _fwd(L, d=96) == _fwd(L)  # head dim 96 runs on the 128-wide kernels
    assert _fwd(L, d=80) == UNSUPPORTED
    if NO_GPU:
        assert _fwd(L, d=256) == _fwd(L)  # head dim 256 has a forward kernel of its own
    assert _fwd(L, d=192) == UNSUPPORTED and _fwd(L, d=512) == UNSUPPORTED
    # Any N >= 1 passes validation (the last 128-row tile may be partial): such a call
    # gets as far as a valid one, which on a machine without a GPU is FA_ERR_CUDA.
    if NO_GPU:
        assert _fwd(L, N=130) == _fwd(L, N=128) not in (INVALID, UNSUPPORTED, ALIGN)
    if NO_GPU:
        assert _fwd(L, N=1) == _fwd(L, N=128)
    assert _fwd(L, B=1 << 16, H=1 << 16, N=128) == UNSUPPORTED  # B*H*N beyond int32
    assert _fwd(L, scale=float("nan")) == INVALID
    assert _fwd(L, scale=float("inf")) == INVALID


def test_cross_argument_checks(L):
    f = L.fa_fwd_qk
    assert f(A, A, A, A, A, 1, 1, 128, 0, 64, 0, 0.1, None) == INVALID
    assert f(A, A, A, A, A, 1, 1, 0, 128, 64, 0, 0.1, None) == INVALID
    assert f(A, A, A, A, A, 1, 1, 128, 256, 80, 0, 0.1, None) == UNSUPPORTED
    if NO_GPU:
        assert f(A, A, A, A, A, 1, 1, 100, 300, 64, 1, 0.1, None) == _fwd(L)  # valid: as far as a square call
    g = L.fa_bwd_qk
    assert g(A, A, A, A, A, A, A, A, A, A, 1 << 20, 1, 1, 128, 0, 64, 0, 0.1, None) == INVALID
    assert g(A, A, A, A, A, A, A, A, A, A, 0, 1, 1, 128, 64, 64, 0, 0.1, None) == WORKSPACE


def test_layout_argument_checks(L):
    f = L.fa_fwd_ex
    assert f(A, A, A, A, A, 1, 1, 128, 128, 64, 2, 0, 0.1, None) == INVALID   # unknown layout
    assert f(A, A, A, A, A, 1, 1, 128, 128, 64, -1, 0, 0.1, None) == INVALID
    if NO_GPU:
        assert f(A, A, A, A, A, 1, 1, 128, 128, 64, 1, 0, 0.1, None) == _fwd(L)  # [B, N, H, d]: valid
    g = L.fa_bwd_ex
    assert g(A, A, A, A, A, A, A, A, A, A, 1 << 20, 1, 1, 128, 128, 64, 3, 0, 0.1, None) == INVALID


def test_blocksparse_argument_checks(L):
    f = L.fa_fwd_blocksparse
    assert f(A, A, A, A, A, None, 128, 1, 1, 128, 64, 0.1, None) == INVALID
    assert f(A, A, A, A, A, A, 64, 1, 1, 128, 64, 0.1, None) == UNSUPPORTED
    assert f(A, A, A, A, A, A, 128, 1, 1, 128, 48, 0.1, None) == UNSUPPORTED


def test_workspace_bytes(L):
    up = lambda x: (x + 255) // 256 * 256
    for (B, H, N, d) in ((1, 1, 128, 64), (8, 16, 2048, 64), (2, 16, 8192, 128), (3, 5, 384, 128)):
        rows = B * H * N
        assert L.fa_bwd_workspace_bytes(B, H, N, d) == 2 * up(rows * 4)
    # N not a multiple of 128: rows are padded to whole tiles per (batch, head).
    for (B, H, N, d) in ((1, 1, 1, 64), (2, 3, 130, 128), (1, 16, 2000, 64)):
        rows = B * H * ((N + 127) // 128 * 128)
        assert L.fa_bwd_workspace_bytes(B, H, N, d) == 2 * up(rows * 4)
    assert L.fa_bwd_workspace_bytes(0, 1, 128, 64) == 0
    assert L.fa_bwd_workspace_bytes(1, 1, -128, 64) == 0


def test_fused_workspace_bytes(L):
    """Row arrays of the deterministic backward, then the fp32 dQ accumulator
    [B*H, Npad, 64 or 128] (d = 96 and 128 share the 128-column width)."""
    up = lambda x: (x + 255) // 256 * 256
    for (B, H, N, d) in ((1, 1, 128, 64), (8, 16, 2048, 64), (2, 16, 8192, 128), (2, 3, 130, 96), (1, 1, 1, 128)):
        rows = B * H * ((N + 127) // 128 * 128)
        dk = 64 if d == 64 else 128
        assert L.fa_bwd_fused_workspace_bytes(B, H, N, d) == 2 * up(rows * 4) + up(rows * dk * 4)
    assert L.fa_bwd_fused_workspace_bytes(0, 1, 128, 64) == 0


def test_fused_argument_checks(L):
    need = L.fa_bwd_fused_workspace_bytes(1, 1, 128, 64)
    det = L.fa_bwd_workspace_bytes(1, 1, 128, 64)
    f = lambda ws=A, wsb=need, mask=None, mb=128, causal=0, Nq=128, Nk=128, d=64, layout=0, dq=A, scale=0.1: \
        L.fa_bwd_fused_ex(A, A, A, A, A, A, dq, A, A, ws, wsb, mask, mb, 1, 1, Nq, Nk, d, layout, causal, scale, None)
    assert f(wsb=det) == WORKSPACE  # the deterministic path's workspace is too small here
    assert f(ws=None) == INVALID and f(ws=A + 16) == ALIGN  # workspace 256-byte aligned
    assert f(dq=None) == INVALID and f(dq=A + 2) == ALIGN
    assert f(mask=A, causal=1) == UNSUPPORTED  # block mask with the causal flag
    assert f(mask=A, mb=64) == UNSUPPORTED
    assert f(mask=A, Nk=256) == UNSUPPORTED  # block mask needs Nq = Nk
    assert f(d=80) == UNSUPPORTED and f(Nq=0) == INVALID and f(layout=5) == INVALID
    assert f(scale=float("nan")) == INVALID
    g = L.fa_bwd_fused
    assert g(A, A, A, A, A, A, A, A, A, A, det, 1, 1, 128, 64, 0, 0.1, None) == WORKSPACE
    pre = L.fa_bwd_fused_preprocess
    assert pre(A, A, A, A, det, 1, 1, 128, 64, None) == WORKSPACE
    assert pre(A, A, A, None, need, 1, 1, 128, 64, None) == INVALID
    main = L.fa_bwd_fused_main
    assert main(A, A, A, A, A, A, A, det, None, 128, 1, 1, 128, 64, 0, 0.1, None) == WORKSPACE
    assert main(A, A, A, A, None, A, A, need, None, 128, 1, 1, 128, 64, 0, 0.1, None) == INVALID
    conv = L.fa_bwd_fused_dq
    assert conv(A, A, det, 1, 1, 128, 64, 0.1, None) == WORKSPACE
    assert conv(None, A, need, 1, 1, 128, 64, 0.1, None) == INVALID
    assert conv(A, A, need, 1, 1, 128, 64, float("inf"), None) == INVALID
    if NO_GPU:  # valid arguments get as far as the first CUDA call, as a forward does
        assert f() == _fwd(L)


def test_merge_forward_and_f32_argument_checks(L):
    m = lambda q=A, oa=A, la=A, d=64, N=128: L.fa_fwd_merge(q, A, A, oa, la, 1, 1, N, d, 0, 0.1, None)
    assert m(oa=None) == INVALID and m(la=None) == INVALID and m(q=None) == INVALID
    assert m(oa=A + 8) == ALIGN
    assert m(d=96) == UNSUPPORTED and m(d=256) == UNSUPPORTED  # merging kernels: head dims 64 and 128
    assert m(N=0) == INVALID
    need = L.fa_bwd_fused_workspace_bytes(1, 1, 128, 64)
    f = lambda dk=A, d=64, wsb=need: L.fa_bwd_fused_main_f32(A, A, A, A, dk, A, A, wsb, 1, 1, 128, d, 0, 0.1, None)
    assert f(dk=None) == INVALID and f(dk=A + 4) == ALIGN
    assert f(wsb=L.fa_bwd_workspace_bytes(1, 1, 128, 64)) == WORKSPACE
    assert f(d=256) == UNSUPPORTED
    acc = L.fa_accumulate_f32
    assert acc(A, A, 12, None) == INVALID and acc(A, A, -8, None) == INVALID
    assert acc(None, A, 8, None) == INVALID and acc(A + 8, A, 8, None) == ALIGN
    assert acc(A, A, 0, None) == OK


def test_dropout_argument_checks(L):
    f = lambda p=0.1, d=64, N=128, q=A: L.fa_fwd_dropout(q, A, A, A, A, 1, 1, N, d, 0, 0.125, p, 5, 0, None)
    b = lambda p=0.1, d=64: L.fa_bwd_dropout(A, A, A, A, A, A, A, A, A, A, 1 << 20, 1, 1, 128, d, 0, 0.125, p, 5,
                                             0, None)
    for bad in (-0.1, 1.0, 2.0, float("nan"), float("inf"), 0.999):  # 0.999: keep threshold rounds to 0
        assert f(p=bad) == INVALID and b(p=bad) == INVALID
    assert f(d=96) == UNSUPPORTED and b(d=96) == UNSUPPORTED
    assert f(d=80) == UNSUPPORTED
    assert f(q=None) == INVALID and f(q=A + 2) == ALIGN
    assert f(N=0) == INVALID
    if NO_GPU:
        assert f() == _fwd(L)  # valid arguments get as far as a plain forward does here
    if NO_GPU:
        assert f(p=0.0) == _fwd(L) and f(p=0.998) == _fwd(L)  # t = 256 and t = 1 are valid


def test_merge_argument_checks(L):
    m = lambda oa=A, la=A, op=A, lp=A, rows=128, d=64: L.fa_merge_partial(oa, la, op, lp, rows, d, None)
    assert m(rows=0) == OK and m(oa=None, rows=0) == OK  # nothing to do
    assert m(rows=-1) == INVALID
    assert m(d=96) == UNSUPPORTED and m(d=32) == UNSUPPORTED
    assert m(oa=None) == INVALID and m(lp=None) == INVALID
    assert m(oa=A + 8) == ALIGN and m(op=A + 4) == ALIGN and m(la=A + 2) == ALIGN
    assert m(rows=1 << 41) == UNSUPPORTED
    acc = L.fa_accumulate_bf16
    assert acc(A, A, 12, 0, None) == INVALID and acc(A, A, -8, 0, None) == INVALID
    assert acc(None, A, 8, 0, None) == INVALID and acc(A + 8, A, 8, 0, None) == ALIGN
    assert acc(A, A, 0, 0, None) == OK
    cv = L.fa_to_bf16
    assert cv(A, A, 7, None) == INVALID and cv(A, None, 8, None) == INVALID and cv(A + 2, A, 8, None) == ALIGN


def test_exp2_diagnostic_argument_checks(L):
    e = L.fa_debug_exp2
    assert e(A, A, -1, 0, None) == INVALID
    assert e(A, A, 16, 2, None) == INVALID  # mode 0 (special-function unit) or 1 (polynomial)
    assert e(None, None, 0, 1, None) == OK  # nothing to do
    assert e(None, A, 16, 0, None) == INVALID


def test_wait_timeout_argument_checks(L):
    f = L.fa_debug_wait_timeout
    assert f(0, A, None) == INVALID
    assert f(-5, None, None) == INVALID
    assert f(100001, A, None) == INVALID
    assert f(1000, A + 2, None) == ALIGN
    g = L.fa_debug_stall_producer
    assert g(2, 1000) == INVALID
    assert g(1, 0) == INVALID
    assert g(1, 100001) == INVALID
    assert g(0, -7) == OK  # off: the limit is ignored


def test_binding_rejects_cpu_tensors():
    q = torch.zeros((1, 1, 128, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fa.forward(q, q, q)
    with pytest.raises(ValueError):
        fa.backward(q, q, q, q, torch.zeros((1, 1, 128)), q)


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(fa, "_lib", None)
    monkeypatch.setenv("FA_LIB", str(tmp_path / "nope.so"))
    with pytest.raises(fa.FAError):
        fa.lib()
