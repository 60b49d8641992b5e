"""GatedDeltaNet step on the GPU (fmoe_gdn_step, through the C ABI) against the fp64
oracle.

Per head: S <- alpha S; u = S k; S <- S + beta (v - u) k^T; o = S q.  The GPU computes
in fp32 (as the pages' single-precision BLAS does); every dot product of length dk is a
chain of four fused multiply-adds per lane and a five-level shuffle tree, whose error is
below about 9 * 2^-24 of the sum of the absolute products.  For these inputs that is
under 1e-5 of the outputs' rms, so the bound here is |gpu - oracle| <= 3e-5 * (|oracle| +
rms(oracle)) per step (and 3e-4 after eight chained steps, the state carrying the
errors forward).
"""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


def _inputs(heads, dk, dv, seed):
    rng = np.random.default_rng(seed)
    S = (0.1 * rng.standard_normal((heads, dv, dk))).astype(np.float32)
    q = rng.standard_normal((heads, dk)).astype(np.float32)
    k = rng.standard_normal((heads, dk)).astype(np.float32)
    q /= np.linalg.norm(q, axis=1, keepdims=True)  # GatedDeltaNet's L2-normalised queries and keys
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((heads, dv)).astype(np.float32)
    alpha = rng.uniform(0.5, 1.0, heads).astype(np.float32)
    beta = rng.uniform(0.0, 1.0, heads).astype(np.float32)
    return S, q.astype(np.float32), k.astype(np.float32), v, alpha, beta


def _dev(*arrays):
    return [torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in arrays]


def _within(got, ref, rel):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = float(np.sqrt(np.mean(ref * ref)))
    bound = rel * (np.abs(ref) + rms)
    ratio = np.abs(got - ref) / np.maximum(bound, 1e-300)
    return bool(np.all(ratio <= 1.0)), float(ratio.max())


@pytest.mark.parametrize("heads,dk,dv", [(64, 128, 128), (3, 36, 50), (2, 512, 7), (5, 4, 1)])
def test_gdn_step_matches_oracle(cuda_lib, heads, dk, dv):
    S, q, k, v, alpha, beta = _inputs(heads, dk, dv, seed=heads * 1000 + dk)
    dS, dq, dk_, dv_, da, db = _dev(S, q, k, v, alpha, beta)
    do = torch.empty(heads, dv, dtype=torch.float32, device="cuda")
    cuda_lib.fmoe_gdn_step(dS, dq, dk_, dv_, da, db, do)
    torch.cuda.synchronize()
    gS, go = dS.cpu().numpy(), do.cpu().numpy()
    for h in range(heads):
        rS, ro = oracle.gdn_step(S[h], q[h], k[h], v[h], float(alpha[h]), float(beta[h]))
        ok, worst = _within(gS[h], rS, 3e-5)
        assert ok, f"head {h}: state worst error/bound {worst:.3f}"
        ok, worst = _within(go[h], ro, 3e-5)
        assert ok, f"head {h}: output worst error/bound {worst:.3f}"


def test_gdn_identity_step_keeps_the_state_exactly(cuda_lib):
    """alpha = 1, beta = 0: the state comes back bit for bit, o = S q."""
    heads, dk, dv = 4, 128, 64
    S, q, k, v, _, _ = _inputs(heads, dk, dv, seed=7)
    dS, dq, dk_, dv_, da, db = _dev(S, q, k, v, np.ones(heads, np.float32), np.zeros(heads, np.float32))
    do = torch.empty(heads, dv, dtype=torch.float32, device="cuda")
    cuda_lib.fmoe_gdn_step(dS, dq, dk_, dv_, da, db, do)
    torch.cuda.synchronize()
    assert np.array_equal(dS.cpu().numpy(), S)
    for h in range(heads):
        ok, worst = _within(do.cpu().numpy()[h], S[h].astype(np.float64) @ q[h].astype(np.float64), 3e-5)
        assert ok, worst


def test_gdn_eight_chained_steps(cuda_lib):
    """The state carried through eight tokens (new q, k, v, gates each token)."""
    heads, dk, dv = 8, 128, 128
    S, *_ = _inputs(heads, dk, dv, seed=11)
    dS = torch.from_numpy(S.copy()).cuda()
    ref = [S[h].astype(np.float64) for h in range(heads)]
    do = torch.empty(heads, dv, dtype=torch.float32, device="cuda")
    for t in range(8):
        _, q, k, v, alpha, beta = _inputs(heads, dk, dv, seed=100 + t)
        dq, dk_, dv_, da, db = _dev(q, k, v, alpha, beta)
        cuda_lib.fmoe_gdn_step(dS, dq, dk_, dv_, da, db, do)
        outs = []
        for h in range(heads):
            ref[h], o = oracle.gdn_step(ref[h], q[h], k[h], v[h], float(alpha[h]), float(beta[h]))
            outs.append(o)
        torch.cuda.synchronize()
        go = do.cpu().numpy()
        for h in range(heads):
            ok, worst = _within(go[h], outs[h], 3e-4)
            assert ok, f"step {t} head {h}: output worst error/bound {worst:.3f}"
    gS = dS.cpu().numpy()
    for h in range(heads):
        ok, worst = _within(gS[h], ref[h], 3e-4)
        assert ok, f"head {h}: final state worst error/bound {worst:.3f}"


def test_gdn_argument_checks(cuda_lib):
    S, q, k, v, alpha, beta = _inputs(2, 128, 8, seed=3)
    dS, dq, dk_, dv_, da, db = _dev(S, q, k, v, alpha, beta)
    do = torch.empty(2, 8, dtype=torch.float32, device="cuda")
    L = cuda_lib.lib()
    ptrs = [t.data_ptr() for t in (dS, dq, dk_, dv_, da, db, do)]
    assert L.fmoe_gdn_step(*ptrs, 0, 128, 8, None) == 0          # no heads: no-op
    assert L.fmoe_gdn_step(*ptrs, 2, 130, 8, None) == 1          # dk not a multiple of 4
    assert L.fmoe_gdn_step(*ptrs, 2, 516, 8, None) == 1          # dk above 512
    assert L.fmoe_gdn_step(None, *ptrs[1:], 2, 128, 8, None) == 1
    torch.cuda.synchronize()
    assert np.array_equal(dS.cpu().numpy(), S)                   # nothing ran
