"""GPU parity of the prologue (jattn_rope_qkv, jattn_quant_fp8) against the
oracle, through the C ABI.

* 16-bit outputs: every element within half a unit in the last place of the
  oracle's FP64 rotation plus the fp32 rotation error bound (a few fp32 ulps
  of the pair's magnitude, which matters only under cancellation), and at
  least 99% of them equal to the exactly rounded value; V exactly equal (a
  conversion).
* e4m3 outputs: codes equal to the oracle's encoding of the same values,
  except where the value sits within 2^-20 of an e4m3 rounding midpoint
  (there an fp32-vs-fp64 last-bit difference may flip the code by one step);
  V codes and all scales of V bit-exact; Q/K scales within 1e-6.
* Standalone quantiser: codes and scales bit-exact (its inputs are exact).
* Query/key RMSNorm fused in front of the rotation (jattn_rope_qkv_norm): the
  same bounds with the fp32 normalisation's error added (sum of 128 squares
  and the hardware 1/sqrt, at most 2 ulp: a few 2^-23 relative, bounded
  here by 2^-18 of the pair's magnitude), and a 2^-17 ambiguity window for
  e4m3 codes.
"""
import numpy as np
import pytest
import torch

import oracle
from diffusion_transformer_joint_jattn_b200 import jattn
from diffusion_transformer_joint_jattn_b200 import workloads as W
from parity_util import to_device

pytestmark = pytest.mark.gpu


def _ulp16(y: np.ndarray, dtype) -> np.ndarray:
    mant = 10 if dtype == torch.float16 else 7
    emin = -14 if dtype == torch.float16 else -126
    e = np.floor(np.log2(np.maximum(np.abs(y), 2.0 ** emin)))
    return 2.0 ** (e - mant)


def _check_rotated(got: torch.Tensor, ref: np.ndarray, dtype, name: str, rel: float = 2.0 ** -20):
    """got: 16-bit [..., d]; ref: float64 exact rotation [..., d]; rel: the
    fp32 arithmetic's error bound relative to the pair's magnitude."""
    g = got.cpu().to(torch.float64).numpy()
    pair = np.sqrt(ref[..., 0::2] ** 2 + ref[..., 1::2] ** 2)
    pair = np.repeat(pair, 2, axis=-1)
    bound = 0.5 * _ulp16(ref, dtype) * (1 + 2.0 ** -10) + rel * pair
    err = np.abs(g - ref)
    assert np.all(err <= bound), f"{name}: {np.sum(err > bound)} elements beyond the bound, worst {np.max(err / bound):.2f}x"
    exact = torch.from_numpy(ref).to(dtype).to(torch.float64).numpy()
    assert np.mean(g != exact) < 0.01, f"{name}: {100 * np.mean(g != exact):.3f}% not exactly rounded"


def _expected_rot(w, inp):
    qr, kr, v = oracle.rotated_qkv(inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"], inp["pos"], w.split, w.theta)
    return qr, kr, v


CASES = [
    dict(B=1, H=2, d=64, S_txt=32, grid=16, n_ref=0),     # the tiny workload
    dict(B=2, H=3, d=128, S_txt=77, grid=9, n_ref=1),     # ragged: S = 77 + 81 + 81 = 239
    dict(B=1, H=1, d=128, S_txt=0, grid=12, n_ref=2),     # no text, two references
    dict(B=1, H=2, d=128, S_txt=5, grid=0, n_ref=0),      # text only, S < 128
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c['B']}H{c['H']}d{c['d']}t{c['S_txt']}g{c['grid']}r{c['n_ref']}")
@pytest.mark.parametrize("out", ["fp16", "bf16"])
def test_rope_16bit_within_one_ulp(cuda_device, case, out):
    w = W.custom(**case)
    inp = W.make_inputs(w, seed=11)
    dinp = to_device(inp, cuda_device)
    q, k, v, sc = jattn.rope_qkv(dinp["qkv_txt"], dinp["qkv_img"], dinp["qkv_ref"], dinp["pos"], w.split,
                                 w.theta, out)
    torch.cuda.synchronize()
    assert sc is None
    qr, kr, vr = _expected_rot(w, inp)
    dt = torch.float16 if out == "fp16" else torch.bfloat16
    for name, got, ref in (("q", q, qr), ("k", k, kr)):
        _check_rotated(got, ref, dt, name)
    assert torch.equal(v.cpu(), torch.from_numpy(vr).to(dt))
    code, bits = jattn.device_status()
    assert code == jattn.OK and bits == 0


@pytest.mark.parametrize("case", CASES[:3], ids=lambda c: f"B{c['B']}H{c['H']}d{c['d']}S{c['S_txt']}")
def test_rope_e4m3_codes_and_scales(cuda_device, case):
    w = W.custom(**case)
    inp = W.make_inputs(w, seed=5)
    dinp = to_device(inp, cuda_device)
    q8, k8, v8, sc = jattn.rope_qkv(dinp["qkv_txt"], dinp["qkv_img"], dinp["qkv_ref"], dinp["pos"], w.split,
                                    w.theta, "e4m3")
    torch.cuda.synchronize()
    qr, kr, vr = _expected_rot(w, inp)
    sc = sc.cpu().numpy()
    for i, (got, ref) in enumerate(((q8, qr), (k8, kr), (v8, vr))):
        x32 = ref.astype(np.float32)
        codes, scales = oracle.quantize_blocks(x32)
        got = got.cpu().view(torch.uint8).numpy()
        if i == 2:       # V is not rotated: its fp32 values are exact on both sides
            np.testing.assert_array_equal(got, codes)
            np.testing.assert_array_equal(sc[2], scales)
            continue
        np.testing.assert_allclose(sc[i], scales, rtol=1e-6)
        inv = 1.0 / np.repeat(sc[i].astype(np.float64), 128, axis=-1)[..., :w.S, None]
        amb = oracle.rounding_ambiguous(x32.astype(np.float64) * inv)
        mism = (got != codes) & ~amb
        assert mism.sum() == 0, f"{mism.sum()} unexplained code mismatches"


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c['B']}H{c['H']}d{c['d']}t{c['S_txt']}g{c['grid']}r{c['n_ref']}")
@pytest.mark.parametrize("out", ["fp16", "bf16"])
def test_rope_norm_16bit(cuda_device, case, out):
    w = W.custom(**case)
    inp = W.make_inputs(w, seed=13)
    nw = W.norm_weights(w.d, 13)
    dinp = to_device(inp, cuda_device)
    q, k, v, _ = jattn.rope_qkv(dinp["qkv_txt"], dinp["qkv_img"], dinp["qkv_ref"], dinp["pos"], w.split, w.theta,
                                out, norm_w=nw.to(cuda_device), eps=1e-6)
    torch.cuda.synchronize()
    qr, kr, vr = oracle.rotated_qkv(inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"], inp["pos"], w.split, w.theta,
                                    norm_w=nw, eps=1e-6)
    dt = torch.float16 if out == "fp16" else torch.bfloat16
    for name, got, ref in (("q", q, qr), ("k", k, kr)):
        _check_rotated(got, ref, dt, name, rel=2.0 ** -18)
    assert torch.equal(v.cpu(), torch.from_numpy(vr).to(dt))
    assert jattn.device_status()[0] == jattn.OK


def test_rope_norm_zero_rows_and_large_eps(cuda_device):
    """An all-zero Q row stays zero (0 * 1/sqrt(eps)); a large eps shrinks the
    result towards zero exactly as the formula says."""
    w = W.custom(B=1, H=2, d=128, S_txt=3, grid=4, n_ref=0)
    inp = W.make_inputs(w, 2)
    inp["qkv_txt"][0, 1, 0, 1] = 0                       # token 1, Q, head 1
    nw = W.norm_weights(128, 2)
    dinp = to_device(inp, cuda_device)
    for eps in (1e-6, 4.0):
        q, k, _, _ = jattn.rope_qkv(dinp["qkv_txt"], dinp["qkv_img"], None, dinp["pos"], w.split, w.theta, "fp16",
                                    norm_w=nw.to(cuda_device), eps=eps)
        torch.cuda.synchronize()
        assert torch.all(q[0, 1, 1].cpu() == 0)
        qr, kr, _ = oracle.rotated_qkv(inp["qkv_txt"], inp["qkv_img"], None, inp["pos"], w.split, w.theta,
                                       norm_w=nw, eps=eps)
        _check_rotated(q, qr, torch.float16, "q", rel=2.0 ** -18)
        _check_rotated(k, kr, torch.float16, "k", rel=2.0 ** -18)


@pytest.mark.parametrize("case", CASES[:3], ids=lambda c: f"B{c['B']}H{c['H']}d{c['d']}S{c['S_txt']}")
def test_rope_norm_e4m3(cuda_device, case):
    w = W.custom(**case)
    inp = W.make_inputs(w, seed=17)
    nw = W.norm_weights(w.d, 17)
    dinp = to_device(inp, cuda_device)
    q8, k8, v8, sc = jattn.rope_qkv(dinp["qkv_txt"], dinp["qkv_img"], dinp["qkv_ref"], dinp["pos"], w.split,
                                    w.theta, "e4m3", norm_w=nw.to(cuda_device), eps=1e-6)
    torch.cuda.synchronize()
    qr, kr, vr = oracle.rotated_qkv(inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"], inp["pos"], w.split, w.theta,
                                    norm_w=nw, eps=1e-6)
    sc = sc.cpu().numpy()
    for i, (got, ref) in enumerate(((q8, qr), (k8, kr), (v8, vr))):
        x32 = ref.astype(np.float32)
        codes, scales = oracle.quantize_blocks(x32)
        got = got.cpu().view(torch.uint8).numpy()
        if i == 2:
            np.testing.assert_array_equal(got, codes)
            np.testing.assert_array_equal(sc[2], scales)
            continue
        np.testing.assert_allclose(sc[i], scales, rtol=2.0 ** -17)
        inv = 1.0 / np.repeat(sc[i].astype(np.float64), 128, axis=-1)[..., :w.S, None]
        amb = oracle.rounding_ambiguous(ref * inv, rel=2.0 ** -17)
        mism = (got != codes) & ~amb
        assert mism.sum() == 0, f"{mism.sum()} unexplained code mismatches"


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("S", [1, 128, 300])
def test_quant_fp8_bit_exact(cuda_device, dtype, S):
    g = torch.Generator().manual_seed(S)
    x = (torch.randn(2, 3, S, 128, generator=g) * torch.rand(2, 3, 1, 1, generator=g) * 50).to(dtype)
    x[0, 0, : min(S, 128)] = 0           # an all-zero block: scale 1, codes 0
    x8, sc = jattn.quant_fp8(x.to(cuda_device))
    torch.cuda.synchronize()
    codes, scales = oracle.quantize_blocks(x.to(torch.float32).numpy())
    np.testing.assert_array_equal(x8.cpu().view(torch.uint8).numpy(), codes)
    np.testing.assert_array_equal(sc.cpu().numpy(), scales)


def test_rope_fp16_range_saturates_and_flags(cuda_device):
    w = W.custom(B=1, H=1, d=128, S_txt=4, grid=0, n_ref=0)
    inp = W.make_inputs(w, 0)
    inp["qkv_txt"][0, 1, 2, 0, 5] = 1.0e5            # V channel beyond the fp16 range
    dinp = to_device(inp, cuda_device)
    jattn.device_status(clear=True)
    q, k, v, _ = jattn.rope_qkv(dinp["qkv_txt"], None, None, dinp["pos"], w.split, w.theta, "fp16")
    code, bits = jattn.device_status(clear=True)
    assert code == jattn.ERR_RANGE and bits & jattn.DEV_RANGE
    assert v[0, 0, 1, 5].item() == 65504.0


@pytest.mark.slow
def test_rope_full_size_2048(cuda_device):
    """Full 2048x2048 Base T2I prologue (S = 16896), sampled tokens: 16-bit
    within one ulp, e4m3 codes as above."""
    w = W.BY_NAME["t2i_2048_base"]
    inp = W.make_inputs(w, 0)
    dinp = to_device(inp, cuda_device)
    q, k, v, _ = jattn.rope_qkv(dinp["qkv_txt"], dinp["qkv_img"], dinp["qkv_ref"], dinp["pos"], w.split,
                                w.theta, "fp16")
    q8, k8, v8, sc = jattn.rope_qkv(dinp["qkv_txt"], dinp["qkv_img"], dinp["qkv_ref"], dinp["pos"], w.split,
                                    w.theta, "e4m3")
    torch.cuda.synchronize()
    toks = W.sample_rows(w.with_batch_heads(B=1, H=1), 512, seed=9)[0, 0]
    qkv = torch.cat([inp["qkv_txt"], inp["qkv_img"]], dim=1)        # [B, S, 3, H, d]
    for b in range(w.B):
        x = qkv[b, toks].to(torch.float64).numpy()                   # [m, 3, H, d]
        pos = inp["pos"][toks].numpy()
        for which, got in ((0, q), (1, k)):
            xr = oracle.rope_rotate(np.transpose(x[:, which], (1, 0, 2)), pos, w.split, w.theta)
            _check_rotated(got[b][:, toks], xr, torch.float16, "qk"[which])
    # full-tensor scale check on V (exact) and Q (rel 1e-6)
    vr = qkv[..., 2, :, :].permute(0, 2, 1, 3).to(torch.float32).numpy()
    _, sv = oracle.quantize_blocks(vr)
    np.testing.assert_array_equal(sc[2].cpu().numpy(), sv)


@pytest.mark.slow
def test_rope_norm_full_size_2048(cuda_device):
    """The fused query/key RMSNorm at the full 2048x2048 size (S = 16896),
    sampled tokens: 16-bit within the norm's bound."""
    w = W.BY_NAME["t2i_2048_base"]
    inp = W.make_inputs(w, 0)
    nw = W.norm_weights(w.d, 0)
    dinp = to_device(inp, cuda_device)
    q, k, v, _ = jattn.rope_qkv(dinp["qkv_txt"], dinp["qkv_img"], dinp["qkv_ref"], dinp["pos"], w.split, w.theta,
                                "fp16", norm_w=nw.to(cuda_device), eps=1e-6)
    torch.cuda.synchronize()
    toks = W.sample_rows(w.with_batch_heads(B=1, H=1), 512, seed=9)[0, 0]
    qkv = torch.cat([inp["qkv_txt"], inp["qkv_img"]], dim=1)
    stream = (toks >= w.S_txt).long().numpy()                           # 0 = txt, 1 = img
    for b in range(w.B):
        x = qkv[b, toks].to(torch.float64).numpy()                      # [m, 3, H, d]
        pos = inp["pos"][toks].numpy()
        for which, got in ((0, q), (1, k)):
            wv = nw.to(torch.float64).numpy()[stream, which]            # [m, d]
            xn = oracle.rms_norm(np.transpose(x[:, which], (1, 0, 2)), wv[None], 1e-6)
            xr = oracle.rope_rotate(xn, pos, w.split, w.theta)
            _check_rotated(got[b][:, toks], xr, torch.float16, "qk"[which], rel=2.0 ** -18)
    assert jattn.device_status()[0] == jattn.OK
