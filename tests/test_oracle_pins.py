"""Pins of the fp64 oracle against facts other than itself (CPU only).

Each test fixes one part of the oracle by a value the Flash-MoE pages print, a
closed form, an invariant, a library routine or brute force, chosen so that a
dropped term, a wrong sign or index, or a transposed operand fails one of them.
"""
import itertools
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import fmoe_synth as synth
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_sizes():
    vals = {}
    with open(os.path.join(GOLDEN, "format_sizes.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, val = line.split()[:2]
            vals[name] = float(val)
    return vals


def _tiny_layer(H=128, I=64, E=8, K=2, bits=4, seed=3):
    shape = synth.LayerShape(H, I, E, K, bits, 1, 0)
    return oracle.synthetic_layer(seed, 0, shape), shape


def _x(H, seed=5):
    return oracle.bf16_to_f64(synth.gen_x_token(seed, 0, H))


# ---------------------------------------------------------------- format ----
def test_record_size_matches_pages():
    """6.75 MB per 4-bit expert (pages) = gate+up+down at hidden 4096 with 64-groups."""
    g = _golden_sizes()
    H = int(g["hidden"])
    rb4 = oracle.record_regions(H, 1024, 4)["size"]
    assert rb4 == 7_077_888
    assert rb4 == g["expert_4bit_size"] * 2 ** 20
    rb2 = oracle.record_regions(H, 1024, 2)["size"]
    assert rb2 == 3_932_160
    # whole-model disk sizes on the pages: experts + non-expert weights, within 3 %
    n = int(g["layers"]) * int(g["experts_per_layer"])
    gib = 2.0 ** 30
    assert abs((n * rb4 / gib + g["non_expert"]) / g["disk_4bit"] - 1) < 0.03
    assert abs((n * rb2 / gib + g["non_expert"]) / g["disk_2bit"] - 1) < 0.03
    # the generator's layout agrees byte for byte
    assert synth.record_bytes(H, 1024, 4) == rb4 and synth.record_bytes(H, 1024, 2) == rb2


@pytest.mark.parametrize("bits", [4, 2])
def test_pack_unpack_roundtrip_every_position(bits):
    H, I = 128, 64
    rng = np.random.default_rng(0)
    per = 32 // bits
    p = synth.gen_expert(1, 0, 0, H, I, bits)
    # codes chosen so that each position in a word holds a different value
    codes = (np.arange(I * H).reshape(I, H) * 7 + 3) % (1 << bits)
    words = np.zeros((I, H // per), dtype=np.uint64)
    for k in range(per):
        words |= codes[:, k::per].astype(np.uint64) << np.uint64(bits * k)
    p.gate_q = words.astype(np.uint32)
    p.up_q = rng.integers(0, 2 ** 32, size=p.up_q.shape, dtype=np.uint64).astype(np.uint32)
    rec = synth.pack_record(p, H, I, bits)
    R = oracle.record_regions(H, I, bits)
    gu = rec[R["gu_q"]:R["gu_q"] + I * 2 * R["qh"]].view(np.uint32).reshape(I, 2, -1)
    assert np.array_equal(oracle.unpack_codes(gu[:, 0, :], bits), codes)
    assert np.array_equal(gu[:, 1, :], p.up_q)


@pytest.mark.parametrize("bits,c", [(4, 0), (4, 9), (4, 15), (2, 0), (2, 3)])
def test_all_codes_c_gives_c_scale_plus_bias(bits, c):
    rows, cols = 4, 256
    per = 32 // bits
    word = 0
    for k in range(per):
        word |= c << (bits * k)
    words = np.full((rows, cols // per), word, dtype=np.uint32)
    rng = np.random.default_rng(1)
    s = synth.bf16_bits(np.abs(rng.standard_normal((rows, cols // 64))) * 0.02)
    b = synth.bf16_bits(rng.standard_normal((rows, cols // 64)) * 0.1)
    sb = s.astype(np.uint32) | (b.astype(np.uint32) << 16)
    W = oracle.dequantise(oracle.unpack_codes(words, bits), sb)
    expect = np.repeat(c * synth.bf16_to_f64(s) + synth.bf16_to_f64(b), 64, axis=1)
    assert np.array_equal(W, expect)


def test_one_hot_x_selects_column():
    lay, sh = _tiny_layer()
    ex = lay.expert(2)
    for j in [0, 1, 63, 64, 127]:
        x = np.zeros(sh.hidden)
        x[j] = 1.0
        assert np.array_equal(ex.Wg @ x, ex.Wg[:, j])
        assert np.array_equal(ex.Wu @ x, ex.Wu[:, j])


def test_constant_codes_gate_closed_form():
    """All codes = c: g_r = sum over groups of (c s_rg + b_rg) * sum(x in group)."""
    H, I, c = 256, 64, 11
    p = synth.gen_expert(2, 0, 0, H, I, 4)
    word = sum(c << (4 * k) for k in range(8))
    p.gate_q[:] = word
    ex = oracle.decode_record(synth.pack_record(p, H, I, 4), H, I, 4)
    x = _x(H)
    s = synth.bf16_to_f64((p.gate_sb & 0xFFFF).astype(np.uint16))
    b = synth.bf16_to_f64((p.gate_sb >> 16).astype(np.uint16))
    xs = x.reshape(-1, 64).sum(axis=1)
    closed = ((c * s + b) * xs[None, :]).sum(axis=1)
    assert np.allclose(ex.Wg @ x, closed, rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- router ----
def test_router_weights_sum_to_one_and_order():
    rng = np.random.default_rng(4)
    for K in [1, 2, 4, 10]:
        l = rng.standard_normal(64) * 1.3
        idx, w = oracle.topk_renorm(l, K)
        assert abs(w.sum() - 1.0) < 1e-15
        assert np.all(np.diff(w) <= 0)
        assert list(idx) == list(np.argsort(-l, kind="stable")[:K])


def test_router_k1_weight_is_one():
    idx, w = oracle.topk_renorm(np.array([0.1, 3.0, -2.0, 0.5]), 1)
    assert list(idx) == [1] and w[0] == 1.0


def test_router_k_equals_e_is_full_softmax():
    l = np.random.default_rng(7).standard_normal(16)
    idx, w = oracle.topk_renorm(l, 16)
    p = scipy.special.softmax(l)
    assert np.allclose(w, p[idx], rtol=1e-14, atol=0)


def test_router_dominant_and_ties():
    l = np.zeros(32)
    l[17] = 50.0
    idx, _ = oracle.topk_renorm(l, 3)
    assert idx[0] == 17 and list(idx[1:]) == [0, 1]       # exact ties: lowest index
    l = np.array([1.0, 2.0, 2.0, 0.5, 2.0])
    idx, w = oracle.topk_renorm(l, 2)
    assert list(idx) == [1, 2] and w[0] == w[1] == 0.5


def test_router_order_follows_exact_probabilities_beyond_underflow():
    """Logits hundreds apart: fp64 probabilities of all but the largest underflow to
    0.0, yet the exact probabilities stay strictly ordered.  The selection must be
    the order of the log-probabilities (scipy's log_softmax, which does not
    underflow), ties to the lower index; the weights are the fp64 ones (1, 0, ...)."""
    l = np.array([-3000.0, 0.0, -900.0, -2000.0, -900.0, -5000.0, -1200.0])
    lp = scipy.special.log_softmax(l)
    want = sorted(range(len(l)), key=lambda e: (-lp[e], e))
    for K in (1, 3, 4, 7):
        idx, w = oracle.topk_renorm(l, K)
        assert list(idx) == want[:K]
        assert w[0] == 1.0 and np.all(w[1:] == 0.0)
    assert want[:4] == [1, 2, 4, 6]


def test_router_topk_is_best_subset_by_brute_force():
    rng = np.random.default_rng(11)
    E = 8
    for K in [1, 2, 3]:
        for _ in range(20):
            l = rng.standard_normal(E)
            idx, w = oracle.topk_renorm(l, K)
            best = max(itertools.combinations(range(E), K), key=lambda S: sum(l[list(S)]))
            assert sorted(idx) == sorted(best)
            p = np.exp(l - l.max())
            assert np.allclose(w, p[idx] / p[idx].sum(), rtol=1e-14)


def test_router_logits_are_matvec():
    H, E = 64, 8
    Wr = synth.gen_router(1, 0, E, H)
    x = _x(H)
    l = oracle.router_logits(x, Wr)
    for e in range(E):
        assert math.isclose(l[e], math.fsum(float(Wr[e, c]) * x[c] for c in range(H)), rel_tol=1e-14, abs_tol=1e-15)


def test_router_bias_is_added():
    """A zero router leaves exactly the bias as logits; a bias large enough to
    dominate moves the selection to its expert (workload of the batched stack: a
    per-expert bias skews expert popularity)."""
    H, E = 64, 8
    x = _x(H)
    b = np.array([0.5, -1.25, 2.0, 0.0, -3.0, 1.5, 0.25, -0.75], dtype=np.float32)
    assert np.array_equal(oracle.router_logits(x, np.zeros((E, H), np.float32), b), b.astype(np.float64))
    Wr = synth.gen_router(1, 0, E, H)
    base = oracle.router_logits(x, Wr)
    skew = np.zeros(E, np.float32)
    skew[5] = 100.0
    lb = oracle.router_logits(x, Wr, skew)
    assert lb[5] == base[5] + 100.0 and np.array_equal(np.delete(lb, 5), np.delete(base, 5))
    assert oracle.topk_renorm(lb, 2)[0][0] == 5


# --------------------------------------------------------- swiglu/combine ----
def test_silu_matches_library():
    t = np.linspace(-30, 30, 1001)
    assert np.allclose(oracle.silu(t), t * scipy.special.expit(t), rtol=1e-14, atol=1e-300)
    assert oracle.silu(np.array([0.0]))[0] == 0.0


def _layer_with(mod):
    H, I, E, K = 128, 64, 8, 2
    recs = synth.gen_layer_records(9, 0, synth.LayerShape(H, I, E, K, 4, 1, 0))
    rb = synth.record_bytes(H, I, 4)
    plains = [synth.gen_expert(9, 0, e, H, I, 4) for e in range(E + 1)]
    for e in range(E + 1):
        mod(e, plains[e])
        recs[e * rb:(e + 1) * rb] = synth.pack_record(plains[e], H, I, 4)
    router = synth.gen_router(9, 0, E, H)
    gs = synth.gen_shared_gate(9, 0, H)
    return oracle.OracleLayer(H, I, E, K, 4, recs, router, gs), H


def test_zero_gate_weights_leave_only_shared():
    def zero_routed_gate(e, p):
        if e < 8:
            p.gate_q[:] = 0
            p.gate_sb[:] = 0
    lay, H = _layer_with(zero_routed_gate)
    x = _x(H)
    r = lay.forward(x)
    sig = oracle.shared_sigma(lay.shared_gate, x)
    assert np.allclose(r.y, x + sig * oracle.expert_ffn(lay.expert(8), x), rtol=0, atol=1e-15)


def test_zero_scale_bias_routed_gives_x_plus_shared():
    def zero_sb(e, p):
        if e < 8:
            p.down_sb[:] = 0
    lay, H = _layer_with(zero_sb)
    x = _x(H)
    r = lay.forward(x)
    assert np.array_equal(r.y, x + r.sigma * oracle.expert_ffn(lay.expert(8), x))


def test_shared_gate_zero_gives_half():
    assert oracle.shared_sigma(np.zeros(64), np.ones(64)) == 0.5


def test_shared_gate_matches_library_sigmoid():
    """sigma = expit(g_s . x): a dot product of ln 3 gives 3/4; random vectors agree
    with the library's logistic function."""
    gs = np.zeros(64)
    gs[3] = math.log(3.0)
    x = np.zeros(64)
    x[3] = 1.0
    assert math.isclose(oracle.shared_sigma(gs, x), 0.75, rel_tol=1e-15)
    rng = np.random.default_rng(9)
    for _ in range(20):
        gs, x = rng.standard_normal(64), rng.standard_normal(64)
        s = math.fsum(float(a) * float(b) for a, b in zip(gs, x))
        assert math.isclose(oracle.shared_sigma(gs, x), float(scipy.special.expit(s)), rel_tol=1e-14)
    # arguments far beyond exp's range: sigma tends to 0 and 1 without overflowing
    for s in (-800.0, -50.0, -3.5, 3.5, 50.0, 800.0, 1e6, -1e6):
        gs, x = np.array([s]), np.array([1.0])
        got = oracle.shared_sigma(gs, x)
        assert math.isclose(got, float(scipy.special.expit(s)), rel_tol=1e-14, abs_tol=1e-300), s


def test_power_of_two_down_scaling_is_exact():
    base, H = _layer_with(lambda e, p: None)

    def times4(e, p):
        s = (p.down_sb & 0xFFFF).astype(np.uint16)
        b = (p.down_sb >> 16).astype(np.uint16)
        s4 = synth.bf16_bits(synth.bf16_to_f64(s) * 4.0)
        b4 = synth.bf16_bits(synth.bf16_to_f64(b) * 4.0)
        p.down_sb[:] = s4.astype(np.uint32) | (b4.astype(np.uint32) << 16)
    scaled, _ = _layer_with(times4)
    x = _x(H)
    a = base.forward(x)
    b = scaled.forward(x)
    assert list(a.idx) == list(b.idx)
    assert np.allclose(b.y - x, 4.0 * (a.y - x), rtol=1e-14, atol=1e-15)


# ------------------------------------------------------------ whole layer ----
def _brute_force_layer(lay, x):
    """Independent naive path: every expert dense (codes read by integer
    division from the generator's plain words, not from the packed record), full
    softmax, mask to the top K, renormalise, sum over all E."""
    H, I, E, K, bits = lay.H, lay.I, lay.E, lay.K, lay.bits
    per = 32 // bits          # codes per word
    base = 2 ** bits          # code c of a word is digit c in base 2^bits

    def dense(e):
        p = synth.gen_expert(3, 0, e, H, I, bits)

        def deq(words, sbs, rows, cols):
            W = np.zeros((rows, cols))
            for r in range(rows):
                for c in range(cols):
                    wd = int(words[r, c // per])
                    q = (wd // (base ** (c % per))) % base
                    pair = int(sbs[r, c // 64])
                    s = synth.bf16_to_f64(np.array([pair % 65536], dtype=np.uint16))[0]
                    b = synth.bf16_to_f64(np.array([pair // 65536], dtype=np.uint16))[0]
                    W[r, c] = q * s + b
            return W
        return deq(p.gate_q, p.gate_sb, I, H), deq(p.up_q, p.up_sb, I, H), deq(p.down_q, p.down_sb, H, I)

    logits = np.array([sum(float(lay.router[e, c]) * x[c] for c in range(H)) for e in range(E)])
    p = np.exp(logits - logits.max())
    p /= p.sum()
    kth = sorted(p, reverse=True)[K - 1]
    mask = p >= kth
    wfull = np.where(mask, p, 0.0)
    wfull /= wfull.sum()
    y = x.copy()
    for e in range(E + 1):
        wt = wfull[e] if e < E else 1.0 / (1.0 + math.exp(-sum(float(lay.shared_gate[c]) * x[c] for c in range(H))))
        if wt == 0.0:
            continue
        Wg, Wu, Wd = dense(e)
        g = Wg @ x
        u = Wu @ x
        h = g / (1.0 + np.exp(-g)) * u
        y = y + wt * (Wd @ h)
    return y, np.nonzero(mask)[0]


@pytest.mark.slow
@pytest.mark.parametrize("bits", [4, 2])
def test_whole_layer_matches_brute_force(bits):
    """The whole layer against the naive path, for 4-bit and 2-bit records (the 2-bit
    case pins the 2-bit region offsets and code order of the packed format)."""
    lay, sh = _tiny_layer(H=64, I=64, E=6, K=2, bits=bits)
    for t in range(2):
        x = oracle.bf16_to_f64(synth.gen_x_token(20, t, sh.hidden))
        r = lay.forward(x)
        yb, sel = _brute_force_layer(lay, x)
        assert sorted(r.idx) == sorted(sel)
        assert np.allclose(r.y, yb, rtol=1e-12, atol=1e-12)


def test_expert_forward_equals_forward_with_its_routing():
    """The split entry point's reference (combine for given routing) reproduces the
    whole layer exactly when handed the layer's own routing."""
    lay, sh = _tiny_layer()
    x = _x(sh.hidden, seed=8)
    r = lay.forward(x)
    assert np.array_equal(lay.expert_forward(x, x, r.idx, r.w, r.sigma), r.y)


# ------------------------------------------------------ pre-norm block ----
def test_block_residual_is_the_unnormalised_input():
    """Experts whose down projections are zero add nothing: the block returns h
    itself (not its normalised copy)."""
    def zero_down(e, p):
        p.down_sb[:] = 0
    lay, H = _layer_with(zero_down)
    h = 3.0 * _x(H)
    r = oracle.block_forward(lay, h)
    assert np.array_equal(r.y, h)


def test_block_update_is_scale_invariant():
    """With eps = 0 the normalised vector of 4h equals that of h exactly, so the
    block's update y - h is the same for h and 4h (the experts see RMSNorm(h), not h),
    and it differs from the update of the layer applied to h directly."""
    lay, _ = _tiny_layer()
    h = 0.37 * _x(128)
    a = oracle.block_forward(lay, h, eps=0.0)
    b = oracle.block_forward(lay, 4.0 * h, eps=0.0)
    assert list(a.idx) == list(b.idx)
    # equal up to the fp64 rounding of adding and removing the residual
    assert np.allclose(a.y - h, b.y - 4.0 * h, rtol=0, atol=1e-14 * np.max(np.abs(4.0 * h)))
    direct = lay.forward(h)
    assert not np.allclose(direct.y - h, a.y - h, rtol=1e-3, atol=0)


# -------------------------------------------------------------- rmsnorm ----
def test_bf16_rounding_matches_torch():
    v = np.random.default_rng(2).standard_normal(5000).astype(np.float32).astype(np.float64)
    v = np.concatenate([v, [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8]])  # exact ties
    tb = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.f64_to_bf16_bits(v), tb)


def test_rmsnorm_constant_and_library():
    h = np.full(256, 3.0)
    n = oracle.bf16_to_f64(oracle.rmsnorm_bf16(h, 0.0))
    assert np.all(n == 1.0)
    rng = np.random.default_rng(3)
    h = oracle.bf16_to_f64(synth.bf16_bits(rng.standard_normal(1024) * 5))
    n = oracle.rmsnorm_bf16(h, 1e-6)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(h), (1024,), eps=1e-6)
    refb = oracle.f64_to_bf16_bits(ref.numpy())
    assert np.mean(n == refb) > 0.999
    assert np.max(np.abs(oracle.bf16_to_f64(n) - oracle.bf16_to_f64(refb))) <= 2 ** -7 * np.max(np.abs(oracle.bf16_to_f64(n)))


def test_rmsnorm_eps_inside_the_root():
    """Where mean(h^2) is of the order of eps, eps decides the result: a constant
    vector a gives a / sqrt(a^2 + eps) (here 2^-10 / sqrt(2^-20 + 2^-20) = 2^-1/2), and
    small random vectors agree with the library routine."""
    a = 2.0 ** -10
    n = oracle.bf16_to_f64(oracle.rmsnorm_bf16(np.full(512, a), 2.0 ** -20))
    assert np.all(n == oracle.bf16_to_f64(oracle.f64_to_bf16_bits(np.array([math.sqrt(0.5)])))[0])
    rng = np.random.default_rng(6)
    h = oracle.bf16_to_f64(synth.bf16_bits(rng.standard_normal(1024) * 1e-3))
    n = oracle.rmsnorm_bf16(h, 1e-6)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(h), (1024,), eps=1e-6)
    refb = oracle.f64_to_bf16_bits(ref.numpy())
    assert np.mean(n == refb) > 0.999


def test_tolerance_helper():
    ref = np.array([1.0, -2.0, 0.0, 4.0])
    rms = math.sqrt(np.mean(ref ** 2))
    ok, worst = oracle.within_tolerance(ref + 2e-3 * (np.abs(ref) + rms) * 0.99, ref, out_bf16=False)
    assert ok and worst < 1.0
    ok, _ = oracle.within_tolerance(ref + np.array([0, 0, 2e-3 * rms * 1.01, 0]), ref, out_bf16=False)
    assert not ok


def test_bf16_rounded_values_always_pass_and_two_ulps_fail():
    """A correctly rounded bf16 output passes the bound whatever its magnitude; an
    output two bf16 ulps off fails wherever |ref| dominates rms."""
    rng = np.random.default_rng(5)
    ref = rng.standard_normal(20000) * np.exp(rng.standard_normal(20000))
    rounded = oracle.bf16_to_f64(oracle.f64_to_bf16_bits(ref))
    assert oracle.within_tolerance(rounded, ref)[0]
    assert oracle.bf16_agreement(rounded, ref) == (1.0, 0.0)
    # the bound before rounding alone would reject some correctly rounded values
    assert not oracle.within_tolerance(rounded, ref, out_bf16=False)[0]
    big = np.argmax(np.abs(ref))
    bad = rounded.copy()
    bad[big] += 4 * oracle.bf16_half_ulp(ref[big])
    assert not oracle.within_tolerance(bad, ref)[0]
    assert oracle.bf16_agreement(bad, ref)[1] == 2.0


def test_bf16_half_ulp_values():
    assert oracle.bf16_half_ulp(1.0) == 2.0 ** -8
    assert oracle.bf16_half_ulp(8.2759) == 2.0 ** -5
    assert oracle.bf16_half_ulp(-0.75) == 2.0 ** -9
    assert oracle.bf16_half_ulp(0.0) == 0.0


def test_golden_tiny_regression():
    """The stored tiny-config routing/output (written by tests/golden/make_golden.py
    from this oracle) is reproduced: guards later edits of the oracle."""
    import json
    with open(os.path.join(GOLDEN, "tiny_seed0.json")) as f:
        g = json.load(f)
    shape = synth.CONFIGS["tiny"]["shape"]
    lay = oracle.synthetic_layer(0, 0, shape)
    for tok in g["tokens"]:
        x = oracle.bf16_to_f64(synth.gen_x_token(0, tok["token"], shape.hidden))
        r = lay.forward(x)
        assert [int(i) for i in r.idx] == tok["idx"]
        assert np.allclose(r.w, tok["w"], rtol=1e-14, atol=0)
        assert np.allclose(r.y, tok["y"], rtol=1e-13, atol=1e-15)


# ------------------------------------------------------------ GatedDeltaNet step ----
def _gdn_case(dv=7, dk=5, seed=0):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((dv, dk)), rng.standard_normal(dk), rng.standard_normal(dk),
            rng.standard_normal(dv))


def test_gdn_identity_and_pure_decay():
    """alpha = 1, beta = 0 leaves the state and reads S q; beta = 0 is a pure decay."""
    S, q, k, v = _gdn_case()
    S1, o1 = oracle.gdn_step(S, q, k, v, 1.0, 0.0)
    assert np.array_equal(S1, S) and np.allclose(o1, S @ q, rtol=1e-15, atol=1e-15)
    S2, o2 = oracle.gdn_step(S, q, k, v, 0.25, 0.0)
    assert np.array_equal(S2, 0.25 * S) and np.allclose(o2, 0.25 * (S @ q), rtol=1e-15, atol=1e-15)


def test_gdn_delta_rule_stores_the_value_at_a_unit_key():
    """With |k| = 1 and beta = 1 the updated state maps k exactly to v (the delta
    rule's defining property), whatever alpha and S."""
    S, q, k, v = _gdn_case(9, 6, 1)
    k = k / np.linalg.norm(k)
    for alpha in (1.0, 0.7, 0.01):
        S1, _ = oracle.gdn_step(S, q, k, v, alpha, 1.0)
        assert np.allclose(S1 @ k, v, rtol=1e-12, atol=1e-12)


def test_gdn_matches_closed_form_and_is_rank_one():
    """S' = alpha S (I - beta k k^T) + beta v k^T (the same update as a matrix product);
    S' - alpha S has rank one; o = S' q.  Also a one-hot key and query select a column."""
    S, q, k, v = _gdn_case(6, 8, 2)
    alpha, beta = 0.83, 0.37
    S1, o1 = oracle.gdn_step(S, q, k, v, alpha, beta)
    closed = alpha * S @ (np.eye(8) - beta * np.outer(k, k)) + beta * np.outer(v, k)
    assert np.allclose(S1, closed, rtol=1e-12, atol=1e-12)
    assert np.linalg.matrix_rank(S1 - alpha * S) == 1
    assert np.allclose(o1, closed @ q, rtol=1e-12, atol=1e-12)
    e = np.zeros(8)
    e[3] = 1.0
    S2, o2 = oracle.gdn_step(S, e, e, v, alpha, beta)
    col = alpha * S[:, 3] + beta * (v - alpha * S[:, 3])
    assert np.allclose(o2, col, rtol=1e-14, atol=1e-14) and np.allclose(S2[:, 3], col, rtol=1e-14, atol=1e-14)


def test_gdn_brute_force_loops():
    """A 3 x 2 head by scalar loops (no library products), two steps in sequence."""
    S, q, k, v = _gdn_case(3, 2, 3)
    Sb = S.copy()
    St = S.copy()
    for step, (alpha, beta) in enumerate([(0.9, 0.5), (0.6, 0.2)]):
        qq, kk, vv = q * (step + 1), k - step, v + step
        St, ot = oracle.gdn_step(St, qq, kk, vv, alpha, beta)
        for i in range(3):
            for j in range(2):
                Sb[i][j] *= alpha
        u = [sum(Sb[i][j] * kk[j] for j in range(2)) for i in range(3)]
        for i in range(3):
            for j in range(2):
                Sb[i][j] += beta * (vv[i] - u[i]) * kk[j]
        ob = [sum(Sb[i][j] * qq[j] for j in range(2)) for i in range(3)]
        assert np.allclose(St, Sb, rtol=1e-13, atol=1e-13) and np.allclose(ot, ob, rtol=1e-13, atol=1e-13)
