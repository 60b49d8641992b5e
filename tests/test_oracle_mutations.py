"""Planted mistakes in the oracle must fail its pins (CPU only).

Each case replaces one step of the fp64 oracle with a plausible wrong version -- a
dropped term, a wrong sign, order or index, a transposed or swapped operand -- and
runs every independent pin of ``test_oracle_pins.py`` against it.  At least one pin
must fail, so that a mistake of that kind in the oracle could not go unnoticed.
The stored-output regression (``test_golden_tiny_regression``) is left out: it was
written by the oracle itself and would catch every change without pinning anything.
The mistakes are planted in the oracle on the CPU only; nothing here touches a GPU.
"""
import importlib.util
import math
import os

import numpy as np
import pytest

import oracle
from oracle import fmoe_oracle as fo

HERE = os.path.dirname(os.path.abspath(__file__))
NOT_INDEPENDENT = {"test_golden_tiny_regression"}


def _pins_module():
    spec = importlib.util.spec_from_file_location("_oracle_pins", os.path.join(HERE, "test_oracle_pins.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _pin_calls(mod):
    """(label, zero-argument callable) for every pin, parametrised ones expanded."""
    calls = []
    for name in sorted(dir(mod)):
        fn = getattr(mod, name)
        if not name.startswith("test_") or not callable(fn) or name in NOT_INDEPENDENT:
            continue
        marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
        if not marks:
            calls.append((name, fn))
            continue
        argnames, values = marks[0].args[0], marks[0].args[1]
        names = [a.strip() for a in argnames.split(",")] if isinstance(argnames, str) else list(argnames)
        for v in values:
            args = v if len(names) > 1 else (v,)
            calls.append((f"{name}{list(args)}", lambda fn=fn, args=args: fn(*args)))
    return calls


# ----------------------------------------------------------------- mistakes --
def _unpack_high_first(words, bits):
    words = np.asarray(words, dtype=np.uint32)
    per, mask = 32 // bits, (1 << bits) - 1
    codes = np.empty(words.shape + (per,), dtype=np.int64)
    for k in range(per):
        codes[..., k] = (words.astype(np.int64) >> (32 - bits * (k + 1))) & mask
    return codes.reshape(words.shape[:-1] + (words.shape[-1] * per,))


def _dequantise_with(transform):
    def deq(codes, sb):
        sb = np.asarray(sb, dtype=np.uint32)
        scale = fo.bf16_to_f64((sb & 0xFFFF).astype(np.uint16))
        bias = fo.bf16_to_f64((sb >> 16).astype(np.uint16))
        return transform(np.asarray(codes).astype(np.float64), scale, bias)
    return deq


def _groups(n, size):
    return np.minimum(np.arange(n) // size, 10 ** 9)


ORIG = {k: getattr(fo, k) for k in ("decode_record", "record_regions", "topk_renorm", "router_logits",
                                     "rmsnorm_bf16", "block_forward", "f64_to_bf16_bits", "shared_sigma")}
ORIG_FORWARD = fo.OracleLayer.forward


def _forward_without(drop_shared=False, drop_resid=False, sigma_for_all=False):
    def forward(self, x, resid=None):
        x = np.asarray(x, dtype=np.float64)
        r = x if resid is None else np.asarray(resid, dtype=np.float64)
        idx, w, sig, l = self.route(x)
        y = np.zeros_like(r) if drop_resid else r.copy()
        for k in range(self.K):
            y = y + (sig if sigma_for_all else w[k]) * fo.expert_ffn(self.expert(int(idx[k])), x)
        if self.has_shared and not drop_shared:
            y = y + sig * fo.expert_ffn(self.expert(self.E), x)
        return fo.LayerResult(y=y, idx=idx, w=w, sigma=sig, logits=l)
    return forward


def _topk_with(key=None, weights=None):
    def topk(l, K):
        p = fo.softmax(l)
        order = sorted(range(len(p)), key=key(p) if key else (lambda e: (-p[e], e)))
        idx = np.array(order[:K], dtype=np.int64)
        w = weights(p, idx, np.asarray(l, dtype=np.float64)) if weights else p[idx] / np.sum(p[idx])
        return idx, w
    return topk


def _rmsnorm_with(denominator):
    def rms(h, eps=1e-6):
        h = np.asarray(h, dtype=np.float64)
        return fo.f64_to_bf16_bits(h / denominator(float(np.sum(h * h)), h.size, eps))
    return rms


def _regions_down_swapped(H, I, bits):
    R = dict(ORIG["record_regions"](H, I, bits))
    R["d_q"], R["d_sb"] = R["d_sb"], R["d_q"]
    return R


def _regions_offsets_from_4bit_rows(H, I, bits):
    """Region offsets laid out as if the rows had 4-bit width (the row sizes stay
    right); identical to the true layout for 4-bit records."""
    R = dict(ORIG["record_regions"](H, I, bits))
    R4 = ORIG["record_regions"](H, I, 4)
    for k in ("gu_q", "gu_sb", "d_q", "d_sb"):
        R[k] = R4[k]
    return R


def _bf16_truncate(v):
    f = np.asarray(v, dtype=np.float64).astype(np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


MUTATIONS = {
    # format / dequantisation
    "codes read high bits first": {"unpack_codes": _unpack_high_first},
    "bias term dropped": {"dequantise": _dequantise_with(
        lambda q, s, b: s[:, _groups(q.shape[1], 64)] * q)},
    "scale and bias halves swapped": {"dequantise": _dequantise_with(
        lambda q, s, b: b[:, _groups(q.shape[1], 64)] * q + s[:, _groups(q.shape[1], 64)])},
    "groups of 32 columns": {"dequantise": _dequantise_with(
        lambda q, s, b: s[:, np.minimum(np.arange(q.shape[1]) // 32, s.shape[1] - 1)] * q
        + b[:, np.minimum(np.arange(q.shape[1]) // 32, s.shape[1] - 1)])},
    "gate and up rows swapped": {"decode_record": lambda rec, H, I, bits: (
        lambda ex: fo.DenseExpert(ex.Wu, ex.Wg, ex.Wd))(ORIG["decode_record"](rec, H, I, bits))},
    "down regions swapped": {"record_regions": _regions_down_swapped},
    "2-bit region offsets computed with 4-bit row bytes": {"record_regions": _regions_offsets_from_4bit_rows},
    # SwiGLU / down
    "silu applied to up": {"expert_ffn": lambda ex, x: ex.Wd @ (
        (ex.Wg @ np.asarray(x, np.float64)) * fo.silu(ex.Wu @ np.asarray(x, np.float64)))},
    "silu sign flipped": {"silu": lambda t: t / (1.0 + np.exp(t))},
    "down matrix transposed": {"expert_ffn": lambda ex, x: ex.Wd.T @ (
        fo.silu(ex.Wg @ np.asarray(x, np.float64)) * (ex.Wu @ np.asarray(x, np.float64)))},
    # routing
    "weights not renormalised": {"topk_renorm": _topk_with(weights=lambda p, idx, l: p[idx])},
    "logits renormalised instead of probabilities": {"topk_renorm": _topk_with(
        weights=lambda p, idx, l: l[idx] / np.sum(l[idx]))},
    "ties to the higher index": {"topk_renorm": _topk_with(key=lambda p: (lambda e: (-p[e], -e)))},
    "smallest K selected": {"topk_renorm": _topk_with(key=lambda p: (lambda e: (p[e], e)))},
    "ranked on fp64 probabilities (underflowed ones tie)": {"topk_renorm": _topk_with()},
    "router bias subtracted": {"router_logits": lambda x, Wr, bias=None: ORIG["router_logits"](
        x, Wr, None if bias is None else -np.asarray(bias))},
    "shared gate sign flipped": {"shared_sigma": lambda gs, x: 1.0 - ORIG["shared_sigma"](gs, x)},
    # combine
    "shared expert dropped": {"OracleLayer.forward": _forward_without(drop_shared=True)},
    "residual dropped": {"OracleLayer.forward": _forward_without(drop_resid=True)},
    "routed experts weighted by the shared gate": {"OracleLayer.forward": _forward_without(sigma_for_all=True)},
    # norm / rounding / block
    "mean of squares not divided by H": {"rmsnorm_bf16": _rmsnorm_with(lambda ss, n, eps: math.sqrt(ss + eps))},
    "eps outside the square root": {"rmsnorm_bf16": _rmsnorm_with(lambda ss, n, eps: math.sqrt(ss / n) + eps)},
    "bf16 rounding by truncation": {"f64_to_bf16_bits": _bf16_truncate},
    "block residual normalised": {"block_forward": lambda layer, h, eps=1e-6: (
        lambda n: layer.forward(n, resid=n))(fo.bf16_to_f64(fo.rmsnorm_bf16(np.asarray(h, np.float64), eps)))},
    "block without the norm": {"block_forward": lambda layer, h, eps=1e-6: layer.forward(
        np.asarray(h, np.float64), resid=np.asarray(h, np.float64))},
    # GatedDeltaNet step
    "delta rule with the sign flipped": {"gdn_step": lambda S, q, k, v, a, b: _gdn_with(S, q, k, v, a, b, sign=-1.0)},
    "key read before the decay": {"gdn_step": lambda S, q, k, v, a, b: _gdn_with(S, q, k, v, a, b, read_first=True)},
    "rank-1 update transposed": {"gdn_step": lambda S, q, k, v, a, b: _gdn_with(S, q, k, v, a, b, transpose=True)},
    "query read from the old state": {"gdn_step": lambda S, q, k, v, a, b: _gdn_with(S, q, k, v, a, b, old_read=True)},
}


def _gdn_with(S, q, k, v, alpha, beta, sign=1.0, read_first=False, transpose=False, old_read=False):
    S0 = np.asarray(S, np.float64)
    S = alpha * S0
    u = (S0 if read_first else S) @ np.asarray(k, np.float64)
    d = sign * (np.asarray(v, np.float64) - u) if sign > 0 else (np.asarray(v, np.float64) + u)
    upd = np.outer(k, d) if transpose and S.shape[0] == S.shape[1] else np.outer(d, k)
    if transpose and S.shape[0] != S.shape[1]:
        upd = np.outer(d[::-1], k)
    Sn = S + beta * upd
    o = (S0 if old_read else Sn) @ np.asarray(q, np.float64)
    return Sn, o


@pytest.fixture(scope="module")
def pins():
    return _pin_calls(_pins_module())


def test_every_pin_passes_unmutated(pins):
    assert len(pins) >= 30
    for label, call in pins:
        call()


@pytest.mark.parametrize("mistake", sorted(MUTATIONS))
def test_planted_mistake_fails_a_pin(mistake, pins, monkeypatch):
    for attr, repl in MUTATIONS[mistake].items():
        if attr.startswith("OracleLayer."):
            monkeypatch.setattr(fo.OracleLayer, attr.split(".", 1)[1], repl)
            continue
        monkeypatch.setattr(fo, attr, repl)
        if hasattr(oracle, attr):
            monkeypatch.setattr(oracle, attr, repl)
    failed = []
    for label, call in pins:
        try:
            call()
        except Exception:  # an assertion, or a shape error from a transposed operand
            failed.append(label)
    assert failed, f"the planted mistake '{mistake}' passes every pin"
