"""The C-ABI library without a GPU: it loads, exports every entry point that
include/jattn.h declares, and rejects invalid arguments synchronously with
the documented status codes (before touching the device).  No call here
reaches a kernel launch."""
import ctypes
import os
import re

import pytest

from diffusion_transformer_joint_jattn_b200 import jattn

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "jattn.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(jattn_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ("jattn_rope_qkv", "jattn_quant_fp8", "jattn_fwd_bf16", "jattn_fwd_fp8"):
        assert name in syms


def test_library_exports_every_declared_symbol():
    lib = jattn.load()
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_status_strings_and_version():
    assert jattn.status_string(jattn.OK) == "ok"
    assert "aligned" in jattn.status_string(jattn.ERR_ALIGNMENT)
    assert jattn.load().jattn_version().decode().count(".") == 2


A = 1 << 20          # a 16-byte aligned fake address: never dereferenced (validation fails first)


def shape(B=1, H=1, St=10, Si=0, Sr=0, d=128):
    return ctypes.byref(jattn.make_shape(B, H, St, Si, Sr, d))


@pytest.mark.parametrize("args,code", [
    (dict(St=0), jattn.ERR_INVALID_ARG),                 # S = 0
    (dict(B=0), jattn.ERR_INVALID_ARG),
    (dict(St=-1, Si=5), jattn.ERR_INVALID_ARG),
    (dict(d=96), jattn.ERR_UNSUPPORTED),
    (dict(d=256), jattn.ERR_UNSUPPORTED),
    (dict(B=300, H=300), jattn.ERR_INVALID_ARG),         # B*H beyond the grid limit
    (dict(St=(1 << 24) + 1), jattn.ERR_INVALID_ARG),     # S beyond 2^24
    (dict(H=65535, St=1 << 24), jattn.ERR_INVALID_ARG),  # 2^16 query-tile pairs x 65535 heads: work items past 2^31
])
def test_fwd_rejects_bad_shapes(args, code):
    lib = jattn.load()
    assert lib.jattn_fwd_bf16(shape(**args), jattn.FP16, A, A, A, A, None, 0.0, None) == code


def test_fwd_rejects_bad_pointers_and_dtypes():
    lib = jattn.load()
    assert lib.jattn_fwd_bf16(shape(), jattn.FP16, None, A, A, A, None, 0.0, None) == jattn.ERR_INVALID_ARG
    assert lib.jattn_fwd_bf16(shape(), jattn.FP16, A + 8, A, A, A, None, 0.0, None) == jattn.ERR_ALIGNMENT
    assert lib.jattn_fwd_bf16(shape(), jattn.FP16, A, A, A, A + 2, None, 0.0, None) == jattn.ERR_ALIGNMENT
    assert lib.jattn_fwd_bf16(shape(), jattn.E4M3, A, A, A, A, None, 0.0, None) == jattn.ERR_UNSUPPORTED
    assert lib.jattn_fwd_bf16(shape(), jattn.FP16, A, A, A, A, A + 1, 0.0, None) == jattn.ERR_ALIGNMENT
    assert lib.jattn_fwd_bf16(shape(), jattn.FP16, A, A, A, A, None, float("nan"), None) == jattn.ERR_INVALID_ARG
    assert lib.jattn_fwd_fp8(shape(), A, A, A, None, A, None, 0.0, None) == jattn.ERR_INVALID_ARG


def _split(*v):
    return (ctypes.c_int32 * 3)(*v)


def test_rope_rejects_bad_arguments():
    lib = jattn.load()
    ok_split = _split(16, 56, 56)
    f = lib.jattn_rope_qkv
    # split must be even, non-negative and sum to d
    assert f(shape(), A, None, None, A, 1e4, _split(16, 56, 58), jattn.FP16, A, A, A, None, None) == jattn.ERR_INVALID_ARG
    assert f(shape(), A, None, None, A, 1e4, _split(15, 57, 56), jattn.FP16, A, A, A, None, None) == jattn.ERR_INVALID_ARG
    # a non-empty stream needs a pointer; theta must be positive
    assert f(shape(Si=4), A, None, None, A, 1e4, ok_split, jattn.FP16, A, A, A, None, None) == jattn.ERR_INVALID_ARG
    assert f(shape(), A, None, None, A, -1.0, ok_split, jattn.FP16, A, A, A, None, None) == jattn.ERR_INVALID_ARG
    # e4m3 output needs a scales buffer
    assert f(shape(), A, None, None, A, 1e4, ok_split, jattn.E4M3, A, A, A, None, None) == jattn.ERR_INVALID_ARG
    # alignment of a stream and of an output
    assert f(shape(), A + 4, None, None, A, 1e4, ok_split, jattn.FP16, A, A, A, None, None) == jattn.ERR_ALIGNMENT
    assert f(shape(), A, None, None, A, 1e4, ok_split, jattn.FP16, A, A + 8, A, None, None) == jattn.ERR_ALIGNMENT
    assert f(shape(), A, None, None, A, 1e4, ok_split, 7, A, A, A, None, None) == jattn.ERR_UNSUPPORTED


def test_rope_norm_rejects_bad_arguments():
    """The RMSNorm variant: weights required, eps > 0 and finite, weights
    16-byte aligned; the shared checks of jattn_rope_qkv still apply."""
    lib = jattn.load()
    ok_split = _split(16, 56, 56)
    f = lib.jattn_rope_qkv_norm
    args = lambda w, eps, sp=ok_split: (shape(), A, None, None, A, 1e4, sp, w, eps, jattn.FP16, A, A, A, None, None)
    assert f(*args(None, 1e-6)) == jattn.ERR_INVALID_ARG
    assert f(*args(A, 0.0)) == jattn.ERR_INVALID_ARG
    assert f(*args(A, -1e-6)) == jattn.ERR_INVALID_ARG
    assert f(*args(A, float("nan"))) == jattn.ERR_INVALID_ARG
    assert f(*args(A, float("inf"))) == jattn.ERR_INVALID_ARG
    assert f(*args(A + 4, 1e-6)) == jattn.ERR_ALIGNMENT
    assert f(*args(A, 1e-6, _split(16, 56, 58))) == jattn.ERR_INVALID_ARG


def test_repair_count_and_workspace_on_the_host():
    """Pure host arithmetic: n = ceil(rho * S - 1e-3) within [0, S]; the
    workspace grows with S and n; invalid arguments give -1 / 0."""
    lib = jattn.load()
    assert lib.jattn_repair_count(shape(B=2, H=24, St=512, Si=16384), 0.005) == 85
    assert lib.jattn_repair_count(shape(St=10), 0.3) == 3
    assert lib.jattn_repair_count(shape(St=10), 0.0) == 0
    assert lib.jattn_repair_count(shape(St=10), 1.0) == 10
    assert lib.jattn_repair_count(shape(St=10), 1.5) == -1
    assert lib.jattn_repair_count(shape(d=96), 0.1) == -1
    w0 = lib.jattn_fwd_fp8_repair_workspace(shape(St=300), 0.0)
    w1 = lib.jattn_fwd_fp8_repair_workspace(shape(St=300), 0.1)
    assert 0 < w0 < w1 and w1 % 256 == 0
    assert lib.jattn_fwd_fp8_repair_workspace(shape(St=300), -0.1) == 0


def test_repair_rejects_bad_arguments():
    lib = jattn.load()
    f = lib.jattn_fwd_fp8_repair
    sp = _split(16, 56, 56)
    need = lib.jattn_fwd_fp8_repair_workspace(shape(), 0.1)

    def call(rho=0.1, ws=A, nbytes=None, o=A, norm=None, eps=1e-6, rep=None, split=sp):
        return f(shape(), A, None, None, A, 1e4, split, norm, eps, rho, ws, need if nbytes is None else nbytes,
                 o, None, rep, 0.0, None)
    assert call(rho=1.5) == jattn.ERR_INVALID_ARG
    assert call(rho=float("nan")) == jattn.ERR_INVALID_ARG
    assert call(ws=None) == jattn.ERR_INVALID_ARG
    assert call(o=None) == jattn.ERR_INVALID_ARG
    assert call(nbytes=need - 1) == jattn.ERR_INVALID_ARG
    assert call(ws=A + 16) == jattn.ERR_ALIGNMENT
    assert call(norm=A, eps=0.0) == jattn.ERR_INVALID_ARG
    assert call(rep=A + 2) == jattn.ERR_ALIGNMENT
    assert call(split=_split(16, 56, 58)) == jattn.ERR_INVALID_ARG


def test_noalloc_refuses_before_launch():
    """The allocation-free entry point: an input whose workspace exceeds the
    library's scratch array is refused on the host, and invalid shapes or
    budgets give the same codes as the workspace entry point."""
    lib = jattn.load()
    f = lib.jattn_fwd_fp8_repair_noalloc
    sp = _split(16, 56, 56)
    big = shape(B=2, H=24, St=512, Si=16384 * 2)            # ~1 GB of workspace
    assert lib.jattn_fwd_fp8_repair_workspace(big, 0.005) > jattn.NOALLOC_SCRATCH_BYTES
    assert f(big, A, A, None, A, 1e4, sp, None, 1e-6, 0.005, A, None, None, 0.0, None) == jattn.ERR_UNSUPPORTED
    assert f(shape(), A, None, None, A, 1e4, sp, None, 1e-6, 1.5, A, None, None, 0.0, None) == jattn.ERR_INVALID_ARG
    assert f(shape(d=96), A, None, None, A, 1e4, sp, None, 1e-6, 0.1, A, None, None, 0.0, None) == jattn.ERR_UNSUPPORTED


def test_host_entry_workspace_and_argument_checks():
    """jattn_joint_attention_host: the workspace size is host arithmetic
    (inputs + laid-out operands + output, 256-byte segments); argument errors
    come back before anything is enqueued."""
    lib = jattn.load()
    ws16 = lib.jattn_joint_attention_host_workspace(shape(B=2, St=100, Si=64), jattn.FP16)
    ws8 = lib.jattn_joint_attention_host_workspace(shape(B=2, St=100, Si=64), jattn.E4M3)
    S, H, d = 164, 1, 128
    assert ws16 >= 2 * S * 3 * H * d * 2 + 3 * 2 * H * S * d * 2 + 2 * S * H * d * 2
    assert 0 < ws8 < ws16 and ws16 % 256 == 0
    assert lib.jattn_joint_attention_host_workspace(shape(d=96), jattn.FP16) == 0
    f = lib.jattn_joint_attention_host
    sp = _split(16, 56, 56)
    need = lib.jattn_joint_attention_host_workspace(shape(), jattn.FP16)
    ok = dict(sh=shape(), t=A, pos=A, split=sp, path=jattn.FP16, o=A, ws=A, n=need, theta=1e4)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["sh"], a["t"], None, None, a["pos"], a["theta"], a["split"], a["path"], a["o"], 0.0, a["ws"],
                 a["n"], None)
    assert call(path=9) == jattn.ERR_UNSUPPORTED
    assert call(sh=shape(d=96)) == jattn.ERR_UNSUPPORTED
    assert call(t=None) == jattn.ERR_INVALID_ARG
    assert call(o=None) == jattn.ERR_INVALID_ARG
    assert call(ws=None) == jattn.ERR_INVALID_ARG
    assert call(n=need - 1) == jattn.ERR_INVALID_ARG
    assert call(ws=A + 16) == jattn.ERR_ALIGNMENT
    assert call(theta=0.0) == jattn.ERR_INVALID_ARG
    assert call(split=_split(16, 56, 58)) == jattn.ERR_INVALID_ARG


def test_quant_rejects_bad_arguments():
    lib = jattn.load()
    f = lib.jattn_quant_fp8
    assert f(shape(), jattn.E4M3, A, A, A, None) == jattn.ERR_UNSUPPORTED
    assert f(shape(), jattn.FP16, A, A, None, None) == jattn.ERR_INVALID_ARG
    assert f(shape(), jattn.FP16, A + 2, A, A, None) == jattn.ERR_ALIGNMENT


def test_selftest_rejects_bad_limit():
    assert jattn.load().jattn_selftest_wait_timeout(0, None) == jattn.ERR_INVALID_ARG


def test_noalloc_scratch_size_matches_the_header():
    """The binding's copy of JATTN_NOALLOC_SCRATCH_BYTES equals the header's
    macro (the oversize tests size their inputs from the binding's copy)."""
    text = open(HEADER).read()
    m = re.search(r"#define\s+JATTN_NOALLOC_SCRATCH_BYTES\s+\(\(size_t\)(\d+)\s*<<\s*(\d+)\)", text)
    assert m is not None
    assert int(m.group(1)) << int(m.group(2)) == jattn.NOALLOC_SCRATCH_BYTES


def test_last_device_status_is_exported():
    lib = jattn.load()
    assert hasattr(lib, "jattn_last_device_status")
    assert "jattn_last_device_status" in declared_symbols()


def test_hp_entry_points_reject_bad_arguments():
    """jattn_rope_qkv_hp / jattn_fwd_bf16_hp: scales, correction rows and
    workspace are required; the workspace must be large enough and 256-byte
    aligned; the shared prologue and forward checks still apply."""
    lib = jattn.load()
    sp = _split(16, 56, 56)
    need = lib.jattn_rope_qkv_hp_workspace(shape(B=2, St=300))
    assert need > 0 and need % 256 == 0
    assert lib.jattn_rope_qkv_hp_workspace(shape(d=96)) == 0
    f = lib.jattn_rope_qkv_hp
    ok = dict(sh=shape(), sc=A, qc=A, kc=A, ws=A, n=lib.jattn_rope_qkv_hp_workspace(shape()), split=sp, norm=None,
              eps=1e-6)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["sh"], A, None, None, A, 1e4, a["split"], a["norm"], a["eps"], A, A, A, a["sc"], a["qc"], a["kc"],
                 a["ws"], a["n"], None)
    assert call(sc=None) == jattn.ERR_INVALID_ARG
    assert call(qc=None) == jattn.ERR_INVALID_ARG
    assert call(kc=None) == jattn.ERR_INVALID_ARG
    assert call(ws=None) == jattn.ERR_INVALID_ARG
    assert call(n=ok["n"] - 1) == jattn.ERR_INVALID_ARG
    assert call(ws=A + 16) == jattn.ERR_ALIGNMENT
    assert call(qc=A + 8) == jattn.ERR_ALIGNMENT
    assert call(norm=A, eps=0.0) == jattn.ERR_INVALID_ARG
    assert call(split=_split(16, 56, 58)) == jattn.ERR_INVALID_ARG
    assert call(sh=shape(d=96)) == jattn.ERR_UNSUPPORTED
    g = lib.jattn_fwd_bf16_hp
    assert g(shape(), A, A, A, None, A, A, A, None, 0.0, None) == jattn.ERR_INVALID_ARG
    assert g(shape(), A, A, A, A, None, A, A, None, 0.0, None) == jattn.ERR_INVALID_ARG
    assert g(shape(), A, A, A, A, A, A + 8, A, None, 0.0, None) == jattn.ERR_ALIGNMENT
    assert g(shape(), None, A, A, A, A, A, A, None, 0.0, None) == jattn.ERR_INVALID_ARG
    assert g(shape(d=96), A, A, A, A, A, A, A, None, 0.0, None) == jattn.ERR_UNSUPPORTED


def test_block_sparse_rejects_bad_arguments():
    lib = jattn.load()
    need = lib.jattn_fwd_block_sparse_workspace(shape(St=300))
    assert need > 0 and need % 256 == 0
    assert lib.jattn_fwd_block_sparse_workspace(shape(d=96)) == 0
    f = lib.jattn_fwd_block_sparse
    n = lib.jattn_fwd_block_sparse_workspace(shape())

    def call(dt=jattn.FP16, tau=1.0, ws=A, nb=n, o=A, kl=None, kc=None, sh=None):
        return f(sh or shape(), dt, A, A, A, tau, ws, nb, o, None, kl, kc, 0.0, None)
    assert call(dt=jattn.E4M3) == jattn.ERR_UNSUPPORTED
    assert call(tau=-1.0) == jattn.ERR_INVALID_ARG
    assert call(tau=float("nan")) == jattn.ERR_INVALID_ARG
    assert call(tau=float("inf")) == jattn.ERR_INVALID_ARG
    assert call(ws=None) == jattn.ERR_INVALID_ARG
    assert call(nb=n - 1) == jattn.ERR_INVALID_ARG
    assert call(ws=A + 16) == jattn.ERR_ALIGNMENT
    assert call(o=None) == jattn.ERR_INVALID_ARG
    assert call(kl=A + 2) == jattn.ERR_ALIGNMENT
    assert call(sh=shape(d=96)) == jattn.ERR_UNSUPPORTED
