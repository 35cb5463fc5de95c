"""Python binding of the jattn C ABI (include/jattn.h).

Argument marshalling only: every step of the joint-attention path runs in the
CUDA kernels of ``libjattn.so``.  PyTorch provides device memory and streams.
There is no CPU fallback: if the library is missing or no GPU is present the
calls raise.

Entry points mirror the C names:
  rope_qkv     joint-sequence assembly + 2D axial RoPE (+ e4m3 quantisation)
  quant_fp8    per-(b, h, 128-token block) e4m3 quantisation
  fwd_bf16     attention forward with 16-bit operands, bf16 output
  fwd_fp8      attention forward with e4m3 operands, bf16 output
  rope_qkv_hp / fwd_bf16_hp   the high-precision 16-bit path (range scales,
               split-precision Q.K^T on the outlier channel pairs)
  joint_attention  the whole path in one call (host or device tensors)
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libjattn.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_ALIGNMENT, ERR_CUDA, ERR_TIMEOUT, ERR_RANGE, ERR_INTERNAL = range(8)
DEV_TIMEOUT, DEV_RANGE, DEV_CHECK = 1, 2, 4
BF16, FP16, E4M3 = 0, 1, 2
BLOCK = 128

_DTYPE_CODE = {torch.bfloat16: BF16, torch.float16: FP16, torch.float8_e4m3fn: E4M3}
_CODE_DTYPE = {BF16: torch.bfloat16, FP16: torch.float16, E4M3: torch.float8_e4m3fn}
_NAME_CODE = {"bf16": BF16, "fp16": FP16, "e4m3": E4M3, "fp8": E4M3}

SYMBOLS = ("jattn_rope_qkv", "jattn_rope_qkv_norm", "jattn_quant_fp8", "jattn_fwd_fp8_repair",
           "jattn_fwd_fp8_repair_workspace", "jattn_repair_count", "jattn_fwd_fp8_repair_noalloc",
           "jattn_joint_attention_host", "jattn_joint_attention_host_workspace", "jattn_fwd_bf16", "jattn_fwd_fp8",
           "jattn_rope_qkv_hp", "jattn_rope_qkv_hp_workspace", "jattn_fwd_bf16_hp",
           "jattn_fwd_block_sparse", "jattn_fwd_block_sparse_workspace",
           "jattn_device_status", "jattn_last_device_status", "jattn_selftest_wait_timeout", "jattn_status_string",
           "jattn_version")


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("S_txt", ctypes.c_int32),
                ("S_img", ctypes.c_int32), ("S_ref", ctypes.c_int32), ("d", ctypes.c_int32)]


class JattnError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} (status {code})")


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libjattn.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise FileNotFoundError(f"{path} is missing: run `python -m diffusion_transformer_joint_jattn_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i32, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
    sp = ctypes.POINTER(Shape)
    lib.jattn_rope_qkv.argtypes = [sp, vp, vp, vp, vp, f32, ctypes.POINTER(i32), i32, vp, vp, vp, vp, vp]
    lib.jattn_rope_qkv_norm.argtypes = [sp, vp, vp, vp, vp, f32, ctypes.POINTER(i32), vp, f32, i32, vp, vp, vp,
                                        vp, vp]
    lib.jattn_quant_fp8.argtypes = [sp, i32, vp, vp, vp, vp]
    lib.jattn_fwd_fp8_repair.argtypes = [sp, vp, vp, vp, vp, f32, ctypes.POINTER(i32), vp, f32, f32, vp,
                                         ctypes.c_size_t, vp, vp, vp, f32, vp]
    lib.jattn_fwd_fp8_repair_workspace.argtypes = [sp, f32]
    lib.jattn_repair_count.argtypes = [sp, f32]
    lib.jattn_joint_attention_host.argtypes = [sp, vp, vp, vp, vp, f32, ctypes.POINTER(i32), i32, vp, f32, vp,
                                               ctypes.c_size_t, vp]
    lib.jattn_joint_attention_host_workspace.argtypes = [sp, i32]
    lib.jattn_fwd_fp8_repair_noalloc.argtypes = [sp, vp, vp, vp, vp, f32, ctypes.POINTER(i32), vp, f32, f32, vp, vp,
                                                 vp, f32, vp]
    lib.jattn_fwd_bf16.argtypes = [sp, i32, vp, vp, vp, vp, vp, f32, vp]
    lib.jattn_rope_qkv_hp.argtypes = [sp, vp, vp, vp, vp, f32, ctypes.POINTER(i32), vp, f32, vp, vp, vp, vp, vp,
                                      vp, vp, ctypes.c_size_t, vp]
    lib.jattn_rope_qkv_hp_workspace.argtypes = [sp]
    lib.jattn_fwd_bf16_hp.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp, f32, vp]
    lib.jattn_fwd_block_sparse.argtypes = [sp, i32, vp, vp, vp, f32, vp, ctypes.c_size_t, vp, vp, vp, vp, f32, vp]
    lib.jattn_fwd_block_sparse_workspace.argtypes = [sp]
    lib.jattn_fwd_fp8.argtypes = [sp, vp, vp, vp, vp, vp, vp, f32, vp]
    lib.jattn_device_status.argtypes = [vp, i32, ctypes.POINTER(ctypes.c_uint32)]
    lib.jattn_last_device_status.argtypes = [vp]
    lib.jattn_selftest_wait_timeout.argtypes = [i32, vp]
    lib.jattn_status_string.argtypes = [i32]
    lib.jattn_status_string.restype = ctypes.c_char_p
    lib.jattn_version.restype = ctypes.c_char_p
    for name in SYMBOLS:
        if name not in ("jattn_status_string", "jattn_version"):
            getattr(lib, name).restype = i32
    lib.jattn_fwd_fp8_repair_workspace.restype = ctypes.c_size_t
    lib.jattn_rope_qkv_hp_workspace.restype = ctypes.c_size_t
    lib.jattn_fwd_block_sparse_workspace.restype = ctypes.c_size_t
    lib.jattn_joint_attention_host_workspace.restype = ctypes.c_size_t
    _lib = lib
    return lib


def status_string(code: int) -> str:
    return load().jattn_status_string(code).decode()


def _check(code: int, where: str):
    if code != OK:
        raise JattnError(code, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(t: torch.Tensor, name: str, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def _dev_shape(t: torch.Tensor, name: str, dtype, shape):
    """``t`` must be a contiguous CUDA tensor of ``dtype`` and ``shape``: the
    C ABI sees only a pointer, so a wrong size would become an out-of-bounds
    device access."""
    _dev(t, name, dtype)
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _check_repair_args(B, H, S, d, n, dev, o, lse, repaired, norm_w):
    """Device, dtype and size checks of the FP8-with-repair outputs and norm
    weights, before the call."""
    for name, t in (("o", o), ("lse", lse), ("repaired", repaired), ("norm_w", norm_w)):
        if t is not None and t.device != dev:
            raise ValueError(f"{name} must be on {dev}, got {t.device}")
    if o is not None:
        _dev_shape(o, "o", torch.bfloat16, (B, S, H, d))
    if lse is not None:
        _dev_shape(lse, "lse", torch.float32, (B, H, S))
    if repaired is not None:
        _dev_shape(repaired, "repaired", torch.int32, (B, H, n))
    if norm_w is not None:
        _dev_shape(norm_w, "norm_w", torch.float32, (3, 2, d))


def _streams(parts):
    """Validate the per-stream QKV tensors [B, S_part, 3, H, d] (bf16, CUDA,
    contiguous, one B / H / d for all) and return (B, H, d, [S_txt, S_img, S_ref])."""
    ref = next((t for t in parts if t is not None), None)
    if ref is None:
        raise ValueError("at least one of qkv_txt, qkv_img, qkv_ref must be given")
    if ref.dim() != 5:
        raise ValueError(f"qkv streams must be [B, S, 3, H, d], got {tuple(ref.shape)}")
    B, _, _, H, d = ref.shape
    lens = []
    for name, t in zip(("qkv_txt", "qkv_img", "qkv_ref"), parts):
        if t is None:
            lens.append(0)
            continue
        _dev(t, name, torch.bfloat16)
        if t.dim() != 5 or t.shape[0] != B or t.shape[2] != 3 or t.shape[3] != H or t.shape[4] != d:
            raise ValueError(f"{name} must be [B, S, 3, H, d], got {tuple(t.shape)}")
        if t.device != ref.device:
            raise ValueError(f"{name} must be on {ref.device}, got {t.device}")
        lens.append(t.shape[1])
    return B, H, d, lens


def _positions(pos, S, dev):
    _dev_shape(pos, "pos", torch.int32, (S, 3))
    if pos.device != dev:
        raise ValueError(f"pos must be on {dev}, got {pos.device}")


def make_shape(B, H, S_txt, S_img, S_ref, d) -> Shape:
    return Shape(B, H, S_txt, S_img, S_ref, d)


def n_blocks(S: int) -> int:
    return -(-S // BLOCK)


def rope_qkv(qkv_txt, qkv_img, qkv_ref, pos, split: Sequence[int], theta: float = 10000.0,
             out_dtype="fp16", out=None, stream=None, norm_w=None, eps: float = 1e-6):
    """Assemble the joint sequence and rotate Q/K (after an RMSNorm of Q and K
    when ``norm_w`` is given: fp32 CUDA [3, 2, d], stream x (Q, K)).

    qkv_*: bf16 CUDA tensors [B, S_part, 3, H, d] (None for an empty stream);
    pos: int32 CUDA [S, 3].  Returns (q, k, v, scales); scales is None unless
    out_dtype is e4m3, then fp32 [3, B, H, ceil(S/128)].
    """
    lib = load()
    parts = [qkv_txt, qkv_img, qkv_ref]
    ref = next(t for t in parts if t is not None)
    B, H, d, lens = _streams(parts)
    S = sum(lens)
    _positions(pos, S, ref.device)
    code = _NAME_CODE[out_dtype] if isinstance(out_dtype, str) else _DTYPE_CODE[out_dtype]
    odt = _CODE_DTYPE[code]
    if out is None:
        dev = ref.device
        q = torch.empty(B, H, S, d, dtype=odt, device=dev)
        k = torch.empty_like(q)
        v = torch.empty_like(q)
        scales = torch.empty(3, B, H, n_blocks(S), dtype=torch.float32, device=dev) if code == E4M3 else None
    else:
        q, k, v, scales = out
        for name, t in (("q", q), ("k", k), ("v", v)):
            _dev_shape(t, name, odt, (B, H, S, d))
        if code == E4M3:
            _dev_shape(scales, "scales", torch.float32, (3, B, H, n_blocks(S)))
    sp = (ctypes.c_int32 * 3)(*[int(x) for x in split])
    shape = make_shape(B, H, lens[0], lens[1], lens[2], d)
    if norm_w is None:
        _check(lib.jattn_rope_qkv(ctypes.byref(shape), _ptr(qkv_txt), _ptr(qkv_img), _ptr(qkv_ref), _ptr(pos),
                                  float(theta), sp, code, _ptr(q), _ptr(k), _ptr(v), _ptr(scales),
                                  _stream(stream)), "jattn_rope_qkv")
    else:
        _dev(norm_w, "norm_w", torch.float32)
        if tuple(norm_w.shape) != (3, 2, d):
            raise ValueError(f"norm_w must be [3, 2, {d}], got {tuple(norm_w.shape)}")
        _check(lib.jattn_rope_qkv_norm(ctypes.byref(shape), _ptr(qkv_txt), _ptr(qkv_img), _ptr(qkv_ref),
                                       _ptr(pos), float(theta), sp, _ptr(norm_w), float(eps), code, _ptr(q),
                                       _ptr(k), _ptr(v), _ptr(scales), _stream(stream)), "jattn_rope_qkv_norm")
    return q, k, v, scales


def quant_fp8(x: torch.Tensor, out=None, stream=None):
    """Per-block e4m3 quantisation of a [B, H, S, d] fp16/bf16 tensor."""
    lib = load()
    _dev(x, "x")
    if x.dim() != 4 or x.dtype not in (torch.bfloat16, torch.float16):
        raise ValueError(f"x must be a bf16 / fp16 [B, H, S, d] tensor, got {x.dtype} {tuple(x.shape)}")
    B, H, S, d = x.shape
    if out is None:
        x8 = torch.empty(B, H, S, d, dtype=torch.float8_e4m3fn, device=x.device)
        scales = torch.empty(B, H, n_blocks(S), dtype=torch.float32, device=x.device)
    else:
        x8, scales = out
        _dev_shape(x8, "x8", torch.float8_e4m3fn, (B, H, S, d))
        _dev_shape(scales, "scales", torch.float32, (B, H, n_blocks(S)))
    shape = make_shape(B, H, S, 0, 0, d)
    _check(lib.jattn_quant_fp8(ctypes.byref(shape), _DTYPE_CODE[x.dtype], _ptr(x), _ptr(x8), _ptr(scales),
                               _stream(stream)), "jattn_quant_fp8")
    return x8, scales


def _fwd_outputs(B, H, S, d, dev, o, lse, want_lse):
    if o is None:
        o = torch.empty(B, S, H, d, dtype=torch.bfloat16, device=dev)
    else:
        _dev_shape(o, "o", torch.bfloat16, (B, S, H, d))
    if lse is None and want_lse:
        lse = torch.empty(B, H, S, dtype=torch.float32, device=dev)
    elif lse is not None:
        _dev_shape(lse, "lse", torch.float32, (B, H, S))
    return o, lse


def fwd_bf16(q, k, v, o=None, lse=None, want_lse=False, softmax_scale: float = 0.0, stream=None):
    """O = softmax(Q K^T * scale) V for fp16/bf16 [B, H, S, d] operands."""
    lib = load()
    if q.dim() != 4:
        raise ValueError(f"q must be [B, H, S, d], got {tuple(q.shape)}")
    B, H, S, d = q.shape
    for n, t in (("q", q), ("k", k), ("v", v)):
        _dev_shape(t, n, q.dtype, (B, H, S, d))
    o, lse = _fwd_outputs(B, H, S, d, q.device, o, lse, want_lse)
    shape = make_shape(B, H, S, 0, 0, d)
    _check(lib.jattn_fwd_bf16(ctypes.byref(shape), _DTYPE_CODE[q.dtype], _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                              _ptr(lse), float(softmax_scale), _stream(stream)), "jattn_fwd_bf16")
    return o, lse


def fwd_fp8(q8, k8, v8, scales, o=None, lse=None, want_lse=False, softmax_scale: float = 0.0, stream=None):
    """Attention forward on e4m3 [B, H, S, d] operands with fp32 block scales
    [3, B, H, ceil(S/128)]."""
    lib = load()
    if q8.dim() != 4:
        raise ValueError(f"q8 must be [B, H, S, d], got {tuple(q8.shape)}")
    B, H, S, d = q8.shape
    for n, t in (("q8", q8), ("k8", k8), ("v8", v8)):
        _dev_shape(t, n, torch.float8_e4m3fn, (B, H, S, d))
    _dev_shape(scales, "scales", torch.float32, (3, B, H, n_blocks(S)))
    o, lse = _fwd_outputs(B, H, S, d, q8.device, o, lse, want_lse)
    shape = make_shape(B, H, S, 0, 0, d)
    _check(lib.jattn_fwd_fp8(ctypes.byref(shape), _ptr(q8), _ptr(k8), _ptr(v8), _ptr(scales), _ptr(o),
                             _ptr(lse), float(softmax_scale), _stream(stream)), "jattn_fwd_fp8")
    return o, lse


CORR_COLS = 16        # columns of one correction row (hi and lo of 8 channels)


def rope_qkv_hp(qkv_txt, qkv_img, qkv_ref, pos, split: Sequence[int], theta: float = 10000.0, out=None,
                workspace=None, stream=None, norm_w=None, eps: float = 1e-6):
    """The high-precision 16-bit prologue (jattn_rope_qkv_hp): fp16 q, k, v
    [B, H, S, d] scaled by powers of two 2^-e per (Q|K|V, b, h, block) --
    e = 0 unless the block reaches past the fp16 range --, the scales 2^e
    fp32 [3, B, H, ceil(S/128)], and the correction rows qc, kc fp16
    [B, H, S, 16] of the 4 channel pairs per (b, h) with the largest
    max|q_pair| * max|k_pair|.  Returns (q, k, v, scales, qc, kc)."""
    lib = load()
    parts = [qkv_txt, qkv_img, qkv_ref]
    ref = next(t for t in parts if t is not None)
    B, H, d, lens = _streams(parts)
    S = sum(lens)
    dev = ref.device
    _positions(pos, S, dev)
    shape = make_shape(B, H, lens[0], lens[1], lens[2], d)
    need = lib.jattn_rope_qkv_hp_workspace(ctypes.byref(shape))
    if out is None:
        q = torch.empty(B, H, S, d, dtype=torch.float16, device=dev)
        out = (q, torch.empty_like(q), torch.empty_like(q),
               torch.empty(3, B, H, n_blocks(S), dtype=torch.float32, device=dev),
               torch.empty(B, H, S, CORR_COLS, dtype=torch.float16, device=dev),
               torch.empty(B, H, S, CORR_COLS, dtype=torch.float16, device=dev))
    q, k, v, scales, qc, kc = out
    for name, t in (("q", q), ("k", k), ("v", v)):
        _dev_shape(t, name, torch.float16, (B, H, S, d))
    _dev_shape(scales, "scales", torch.float32, (3, B, H, n_blocks(S)))
    _dev_shape(qc, "qc", torch.float16, (B, H, S, CORR_COLS))
    _dev_shape(kc, "kc", torch.float16, (B, H, S, CORR_COLS))
    if norm_w is not None:
        _dev_shape(norm_w, "norm_w", torch.float32, (3, 2, d))
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    _dev(workspace, "workspace", torch.uint8)
    if workspace.numel() < need:
        raise ValueError(f"workspace must hold at least {need} bytes, got {workspace.numel()}")
    sp = (ctypes.c_int32 * 3)(*[int(x) for x in split])
    _check(lib.jattn_rope_qkv_hp(ctypes.byref(shape), _ptr(qkv_txt), _ptr(qkv_img), _ptr(qkv_ref), _ptr(pos),
                                 float(theta), sp, _ptr(norm_w), float(eps), _ptr(q), _ptr(k), _ptr(v),
                                 _ptr(scales), _ptr(qc), _ptr(kc), _ptr(workspace), workspace.numel(),
                                 _stream(stream)), "jattn_rope_qkv_hp")
    return q, k, v, scales, qc, kc


def rope_qkv_hp_workspace_bytes(B: int, H: int, S_txt: int, S_img: int, S_ref: int, d: int) -> int:
    return load().jattn_rope_qkv_hp_workspace(ctypes.byref(make_shape(B, H, S_txt, S_img, S_ref, d)))


def fwd_bf16_hp(q, k, v, scales, qc, kc, o=None, lse=None, want_lse=False, softmax_scale: float = 0.0,
                stream=None):
    """The high-precision 16-bit forward (jattn_fwd_bf16_hp) on the operands
    rope_qkv_hp wrote."""
    lib = load()
    if q.dim() != 4:
        raise ValueError(f"q must be [B, H, S, d], got {tuple(q.shape)}")
    B, H, S, d = q.shape
    for n, t in (("q", q), ("k", k), ("v", v)):
        _dev_shape(t, n, torch.float16, (B, H, S, d))
    _dev_shape(scales, "scales", torch.float32, (3, B, H, n_blocks(S)))
    _dev_shape(qc, "qc", torch.float16, (B, H, S, CORR_COLS))
    _dev_shape(kc, "kc", torch.float16, (B, H, S, CORR_COLS))
    o, lse = _fwd_outputs(B, H, S, d, q.device, o, lse, want_lse)
    shape = make_shape(B, H, S, 0, 0, d)
    _check(lib.jattn_fwd_bf16_hp(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(scales), _ptr(qc), _ptr(kc),
                                 _ptr(o), _ptr(lse), float(softmax_scale), _stream(stream)), "jattn_fwd_bf16_hp")
    return o, lse


def fwd_block_sparse(q, k, v, tau: float, o=None, lse=None, want_lse: bool = False, want_blocks: bool = False,
                     workspace=None, softmax_scale: float = 0.0, stream=None):
    """Block-sparse attention forward (jattn_fwd_block_sparse) on fp16/bf16
    [B, H, S, d] operands: per 256-row query block, only the 128-key blocks
    whose estimated attention share reaches tau / n_kb (and the largest).
    Returns o (and lse; and, with want_blocks, kv_list int32 [B, H, n_qb,
    n_kb] and kv_count int32 [B, H, n_qb])."""
    lib = load()
    if q.dim() != 4:
        raise ValueError(f"q must be [B, H, S, d], got {tuple(q.shape)}")
    B, H, S, d = q.shape
    for n, t in (("q", q), ("k", k), ("v", v)):
        _dev_shape(t, n, q.dtype, (B, H, S, d))
    o, lse = _fwd_outputs(B, H, S, d, q.device, o, lse, want_lse)
    shape = make_shape(B, H, S, 0, 0, d)
    need = lib.jattn_fwd_block_sparse_workspace(ctypes.byref(shape))
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _dev(workspace, "workspace", torch.uint8)
    if workspace.numel() < need:
        raise ValueError(f"workspace must hold at least {need} bytes, got {workspace.numel()}")
    n_qb, n_kb = -(-S // (2 * BLOCK)), n_blocks(S)
    kv_list = kv_count = None
    if want_blocks:
        kv_list = torch.empty(B, H, n_qb, n_kb, dtype=torch.int32, device=q.device)
        kv_count = torch.empty(B, H, n_qb, dtype=torch.int32, device=q.device)
    _check(lib.jattn_fwd_block_sparse(ctypes.byref(shape), _DTYPE_CODE[q.dtype], _ptr(q), _ptr(k), _ptr(v),
                                      float(tau), _ptr(workspace), workspace.numel(), _ptr(o), _ptr(lse),
                                      _ptr(kv_list), _ptr(kv_count), float(softmax_scale), _stream(stream)),
           "jattn_fwd_block_sparse")
    out = [o]
    if want_lse:
        out.append(lse)
    if want_blocks:
        out += [kv_list, kv_count]
    return out[0] if len(out) == 1 else tuple(out)


def device_status(clear: bool = True, stream=None):
    """(status code, raw bits) of the current device's status word."""
    lib = load()
    bits = ctypes.c_uint32(0)
    code = lib.jattn_device_status(_stream(stream), int(clear), ctypes.byref(bits))
    return code, bits.value


def last_device_status(stream=None) -> int:
    """jattn_last_device_status: wait for ``stream``'s work, return the
    device status word's code without clearing it."""
    return load().jattn_last_device_status(_stream(stream))


def selftest_wait_timeout(limit_ms: int = 50, stream=None):
    _check(load().jattn_selftest_wait_timeout(int(limit_ms), _stream(stream)), "jattn_selftest_wait_timeout")


def repair_count(B: int, H: int, S_txt: int, S_img: int, S_ref: int, d: int, rho: float) -> int:
    """Tokens repaired per (b, h) for budget rho (jattn_repair_count)."""
    n = load().jattn_repair_count(ctypes.byref(make_shape(B, H, S_txt, S_img, S_ref, d)), float(rho))
    if n < 0:
        raise ValueError("invalid shape or rho")
    return n


def repair_workspace_bytes(B: int, H: int, S_txt: int, S_img: int, S_ref: int, d: int, rho: float) -> int:
    return load().jattn_fwd_fp8_repair_workspace(ctypes.byref(make_shape(B, H, S_txt, S_img, S_ref, d)),
                                                 float(rho))


def fwd_fp8_repair(qkv_txt, qkv_img, qkv_ref, pos, split: Sequence[int], theta: float = 10000.0,
                   rho: float = 0.005, norm_w=None, eps: float = 1e-6, want_lse: bool = False,
                   want_repaired: bool = False, softmax_scale: float = 0.0, workspace=None, o=None, lse=None,
                   stream=None):
    """The FP8 path with token repair in one call (jattn_fwd_fp8_repair).

    Returns o bf16 [B, S, H, d], plus lse fp32 [B, H, S] and / or the
    repaired token indices int32 [B, H, n] when asked for.  ``workspace``: a
    uint8 CUDA tensor of at least repair_workspace_bytes(...) bytes (allocated
    here when None)."""
    lib = load()
    parts = [qkv_txt, qkv_img, qkv_ref]
    ref = next(t for t in parts if t is not None)
    B, H, d, lens = _streams(parts)
    S = sum(lens)
    dev = ref.device
    _positions(pos, S, dev)
    n = repair_count(B, H, *lens, d, rho)
    need = repair_workspace_bytes(B, H, *lens, d, rho)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    if o is None:
        o = torch.empty(B, S, H, d, dtype=torch.bfloat16, device=dev)
    if want_lse and lse is None:
        lse = torch.empty(B, H, S, dtype=torch.float32, device=dev)
    rep = torch.empty(B, H, n, dtype=torch.int32, device=dev) if want_repaired else None
    _check_repair_args(B, H, S, d, n, dev, o, lse, rep, norm_w)
    _dev(workspace, "workspace", torch.uint8)
    if workspace.numel() < need:
        raise ValueError(f"workspace must hold at least {need} bytes, got {workspace.numel()}")
    sp = (ctypes.c_int32 * 3)(*[int(x) for x in split])
    shape = make_shape(B, H, lens[0], lens[1], lens[2], d)
    _check(lib.jattn_fwd_fp8_repair(ctypes.byref(shape), _ptr(qkv_txt), _ptr(qkv_img), _ptr(qkv_ref), _ptr(pos),
                                    float(theta), sp, _ptr(norm_w), float(eps), float(rho), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _ptr(o), _ptr(lse),
                                    _ptr(rep if rep is not None and rep.numel() else None), float(softmax_scale),
                                    _stream(stream)), "jattn_fwd_fp8_repair")
    out = [o]
    if want_lse:
        out.append(lse)
    if want_repaired:
        out.append(rep)
    return out[0] if len(out) == 1 else tuple(out)


NOALLOC_SCRATCH_BYTES = 640 << 20


def fwd_fp8_repair_noalloc(qkv_txt, qkv_img, qkv_ref, pos, split: Sequence[int], o, theta: float = 10000.0,
                           rho: float = 0.005, norm_w=None, eps: float = 1e-6, lse=None, repaired=None,
                           softmax_scale: float = 0.0, stream=None):
    """jattn_fwd_fp8_repair_noalloc: the FP8-with-repair path with the
    library's own device scratch.  The caller passes every output buffer
    (o bf16 [B, S, H, d]; optional lse fp32 [B, H, S] and repaired int32
    [B, H, n]); nothing is allocated here or in the library."""
    lib = load()
    parts = [qkv_txt, qkv_img, qkv_ref]
    ref = next(t for t in parts if t is not None)
    B, H, d, lens = _streams(parts)
    S = sum(lens)
    _positions(pos, S, ref.device)
    n = repair_count(B, H, *lens, d, rho)
    if o is None:
        raise ValueError("o must be given: this entry point allocates nothing")
    _check_repair_args(B, H, S, d, n, ref.device, o, lse, repaired, norm_w)
    if repaired is not None and n == 0:
        repaired = None
    sp = (ctypes.c_int32 * 3)(*[int(x) for x in split])
    shape = make_shape(B, H, lens[0], lens[1], lens[2], d)
    _check(lib.jattn_fwd_fp8_repair_noalloc(ctypes.byref(shape), _ptr(qkv_txt), _ptr(qkv_img), _ptr(qkv_ref),
                                            _ptr(pos), float(theta), sp, _ptr(norm_w), float(eps), float(rho), _ptr(o),
                                            _ptr(lse), _ptr(repaired), float(softmax_scale), _stream(stream)),
           "jattn_fwd_fp8_repair_noalloc")
    return o


def joint_attention(qkv_txt, qkv_img, qkv_ref, pos, split, theta: float = 10000.0, path: str = "bf16",
                    operand_dtype: str | None = None, want_lse: bool = False, out=None, stream=None,
                    norm_w=None, eps: float = 1e-6, workspace=None, precise: bool = True):
    """The whole hot path, with the query/key RMSNorm fused into the
    prologue when ``norm_w`` is given.  path "bf16": the high-precision pair
    rope_qkv_hp -> fwd_bf16_hp by default; ``precise=False`` selects the
    plain pair rope_qkv -> fwd_bf16 with ``operand_dtype`` operands ("fp16"
    unless given).  path "fp8": rope_qkv e4m3 -> fwd_fp8.

    CUDA tensors: the device entry points, asynchronous on ``stream``.
    CPU tensors (pinned for overlap): jattn_joint_attention_host, which
    copies in, runs the path and copies O out pipelined over (batch entry,
    head group) chunks; the result lands in ``out`` (a bf16 [B, S, H, d] host
    tensor, allocated here if None) and the call returns once it is there.
    Its plain 16-bit path takes bf16 operands (fp16 operands are those of the
    high-precision pair).  The host entry has no LSE output and no norm;
    those need device tensors.
    Returns O bf16 [B, S, H, d] (and LSE for device tensors)."""
    parts = [qkv_txt, qkv_img, qkv_ref]
    ref = next(t for t in parts if t is not None)
    if not ref.is_cuda:
        if want_lse or norm_w is not None:
            raise ValueError("LSE output and the query/key norm need device tensors")
        lib = load()
        B, _, _, H, d = ref.shape
        lens = [0 if t is None else t.shape[1] for t in parts]
        for name, t in zip(("qkv_txt", "qkv_img", "qkv_ref"), parts):
            if t is not None and (t.dtype != torch.bfloat16 or not t.is_contiguous()):
                raise ValueError(f"{name} must be a contiguous bf16 tensor")
        if pos.dtype != torch.int32 or not pos.is_contiguous():
            raise ValueError("pos must be a contiguous int32 tensor")
        S = sum(lens)
        if path not in ("bf16", "fp8"):
            raise ValueError(f"unknown path {path!r}")
        if path == "fp8":
            code = E4M3
        elif precise:
            code = FP16                   # the host entry's high-precision pair
        elif operand_dtype in (None, "bf16"):
            code = BF16
        else:
            raise ValueError("the host entry's plain 16-bit path takes bf16 operands")
        shape = make_shape(B, H, lens[0], lens[1], lens[2], d)
        need = lib.jattn_joint_attention_host_workspace(ctypes.byref(shape), code)
        dev = torch.device("cuda", torch.cuda.current_device())
        if workspace is None or workspace.numel() * workspace.element_size() < need:
            workspace = torch.empty(need, dtype=torch.uint8, device=dev)
        if out is None:
            out = torch.empty(B, S, H, d, dtype=torch.bfloat16).pin_memory()
        sp = (ctypes.c_int32 * 3)(*[int(x) for x in split])
        st = torch.cuda.current_stream() if stream is None else stream
        _check(lib.jattn_joint_attention_host(ctypes.byref(shape), _ptr(qkv_txt), _ptr(qkv_img), _ptr(qkv_ref),
                                              _ptr(pos), float(theta), sp, code, _ptr(out), 0.0, _ptr(workspace),
                                              workspace.numel() * workspace.element_size(),
                                              ctypes.c_void_p(st.cuda_stream)), "jattn_joint_attention_host")
        st.synchronize()
        return out
    if path == "bf16" and precise:
        q, k, v, sc, qc, kc = rope_qkv_hp(*parts, pos, split, theta, stream=stream, norm_w=norm_w, eps=eps)
        o, lse = fwd_bf16_hp(q, k, v, sc, qc, kc, want_lse=want_lse, stream=stream)
    elif path == "bf16":
        q, k, v, _ = rope_qkv(*parts, pos, split, theta, operand_dtype or "fp16", stream=stream, norm_w=norm_w,
                              eps=eps)
        o, lse = fwd_bf16(q, k, v, want_lse=want_lse, stream=stream)
    elif path == "fp8":
        q, k, v, sc = rope_qkv(*parts, pos, split, theta, "e4m3", stream=stream, norm_w=norm_w, eps=eps)
        o, lse = fwd_fp8(q, k, v, sc, want_lse=want_lse, stream=stream)
    else:
        raise ValueError(f"unknown path {path!r}")
    return (o, lse) if want_lse else o


def flops(B: int, H: int, S: int, d: int) -> int:
    """Algorithmic FLOPs of one attention call: 4 * B * H * S^2 * d."""
    return 4 * B * H * S * S * d


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)
