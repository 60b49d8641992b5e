"""The seeded input generator: published SplitMix64 values, series accuracy,
and bit equality of its host (numpy) and compiled implementations."""
import ctypes
import math

import numpy as np
import pytest
import torch

import fmoe_synth as synth


def test_splitmix64_published_sequence():
    # SplitMix64 seeded with 0: the first three outputs, as published with the
    # reference implementation (Steele et al. 2014; Vigna's splitmix64.c).
    g = synth.GAMMA
    got = [synth.mix64_int((k * g) & synth.MASK64) for k in (1, 2, 3)]
    assert got == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]
    d = synth.draws(0, 0, 3)
    assert [int(v) for v in d] == got


def test_series_ln_cos_accuracy():
    u = np.concatenate([np.linspace(0, 1, 200001)[1:], [2.0 ** -53, 1e-300, 0.5, 0.75]])
    assert np.max(np.abs(synth._ln_unit(u) - np.log(u)) / np.abs(np.log(u) - 1e-300)) < 1e-15
    assert np.max(np.abs(synth._cos_2pi(u) - np.cos(2 * np.pi * u))) < 2e-15


def test_normals_statistics():
    n = synth.normals(synth.stream_key(0, 0, 0, 0), 0, 400000)
    assert abs(n.mean()) < 0.01 and abs(n.std() - 1) < 0.01
    # P(|z| > 2) of the standard normal
    assert abs(np.mean(np.abs(n) > 2) - 0.0455) < 0.003


def test_bf16_matches_torch():
    v = np.random.default_rng(0).standard_normal(20000).astype(np.float32)
    tb = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(synth.bf16_bits(v.astype(np.float64)), tb)


def test_x_is_rms_normalised():
    x = synth.bf16_to_f64(synth.gen_x_token(0, 3, 4096))
    assert abs(math.sqrt(np.mean(x * x)) - 1) < 2e-3


def _host_lib():
    from fmoe_synth import device
    from fmoe_synth.build import build
    build()
    return device.lib()


def test_compiled_generator_host_path_matches_numpy():
    L = _host_lib()
    key = synth.stream_key(7, 2, 5, synth.T_DOWN_SB)
    n = 5000
    out = np.zeros(n, dtype=np.float64)
    L.fmoe_synth_host_normals(out.ctypes.data, key, 123, n)
    assert np.array_equal(out, synth.normals(key, 123, n))
    for (H, I, bits) in [(128, 64, 4), (64, 64, 2), (512, 128, 4)]:
        rb = synth.record_bytes(H, I, bits)
        assert L.fmoe_synth_record_bytes(H, I, bits) == rb
        rec = np.zeros(rb, dtype=np.uint8)
        L.fmoe_synth_host_record(rec.ctypes.data, H, I, bits, 11, 3, 4)
        assert np.array_equal(rec, synth.gen_record(11, 3, 4, H, I, bits))


@pytest.mark.gpu
def test_device_generator_matches_numpy():
    from fmoe_synth import device
    from fmoe_synth.build import build
    build()
    H, I, bits, E = 512, 128, 4, 3
    rb = synth.record_bytes(H, I, bits)
    d = torch.empty(E * rb, dtype=torch.uint8, device="cuda")
    device.fill_records(d, H, I, bits, 0, 1, 5, E)
    got = d.cpu().numpy()
    for e in range(E):
        assert np.array_equal(got[e * rb:(e + 1) * rb], synth.gen_record(0, 1, 5 + e, H, I, bits))
    r = torch.empty(8, H, dtype=torch.float32, device="cuda")
    device.fill_router(r, 0, 1, 8, H)
    assert np.array_equal(r.cpu().numpy(), synth.gen_router(0, 1, 8, H))
    x = torch.empty(4, 4096, dtype=torch.int16, device="cuda")
    device.fill_x(x, 0, 10, 4, 4096)
    assert np.array_equal(x.cpu().numpy().view(np.uint16), synth.gen_x(0, 10, 4, 4096))
