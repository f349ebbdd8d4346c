"""Pins of the Mamba-2 SSD form of Swimba's scan (oracle/swimba_ssd_oracle.py) against facts that
do not come from it: a brute-force unrolled sum, the layer oracle's already-pinned selective scan
(one channel per head), identical experts, superposition, and the chunked form against the
sequential one."""
import itertools

import numpy as np
import pytest

from oracle import swimba_oracle as O
from oracle import swimba_ssd_oracle as SSD

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def ssd_inputs(L=7, k=2, H=3, P=2, N=4, seed=0):
    g = np.random.default_rng(seed)
    w = g.uniform(0.2, 1.0, (L, k))
    return {
        "X": g.standard_normal((L, k, H, P)),
        "B": g.standard_normal((L, k, N)),
        "C": g.standard_normal((L, k, N)),
        "gates": w / w.sum(axis=1, keepdims=True),
        "delta": np.exp(g.uniform(np.log(1e-2), np.log(0.5), (L, H))),
        "A": -np.exp(g.uniform(np.log(0.3), np.log(4.0), H)),
        "D_skip": g.standard_normal(H),
        "S0": 0.5 * g.standard_normal((H, P, N)),
    }


@pytest.mark.parametrize("L", [1, 2, 5])
def test_ssd_brute_force_unrolled_sum(L):
    a = ssd_inputs(L=L, seed=L)
    y, S = SSD.ssd_scan_sequential(**a)
    X, B, C, g, dl, A, Dk, S0 = (a[n] for n in ("X", "B", "C", "gates", "delta", "A", "D_skip", "S0"))
    k, H, P = X.shape[1:]
    for t, h, p in itertools.product(range(L), range(H), range(P)):
        cm = sum(g[t, j] * C[t, j] for j in range(k))
        decay_all = np.prod([np.exp(dl[r, h] * A[h]) for r in range(t + 1)])
        ref = decay_all * float(cm @ S0[h, p])
        for s in range(t + 1):
            decay = np.prod([np.exp(dl[r, h] * A[h]) for r in range(s + 1, t + 1)])
            for j in range(k):
                ref += decay * dl[s, h] * g[s, j] * X[s, j, h, p] * float(cm @ B[s, j])
        ref += Dk[h] * sum(g[t, j] * X[t, j, h, p] for j in range(k))
        assert y[t, h, p] == pytest.approx(ref, rel=1e-12, abs=1e-12)
    # the final state, unrolled
    for h, p, n in itertools.product(range(H), range(P), range(B.shape[2])):
        ref = np.prod(np.exp(dl[:, h] * A[h])) * S0[h, p, n]
        for s in range(L):
            decay = np.prod([np.exp(dl[r, h] * A[h]) for r in range(s + 1, L)])
            ref += decay * dl[s, h] * sum(g[s, j] * X[s, j, h, p] * B[s, j, n] for j in range(k))
        assert S[h, p, n] == pytest.approx(ref, rel=1e-12, abs=1e-12)


def test_one_channel_per_head_reduces_to_the_selective_scan():
    """k = 1, P = 1: head h is channel d = h with A[d, n] = A_h for every n -- the layer oracle's
    selective scan (pinned on its own) with E = 1."""
    L, H, N = 9, 5, 4
    a = ssd_inputs(L=L, k=1, H=H, P=1, N=N, seed=3)
    y, S = SSD.ssd_scan_sequential(**a)
    x = a["X"][:, 0, :, 0][None]  # [1, L, D]
    dt_mix = np.log(np.expm1(a["delta"]))[None]  # softplus(dt_mix) = delta
    Bm, Cm = a["B"][:, 0][None], a["C"][:, 0][None]
    idx = np.zeros((1, L, 1), dtype=np.int32)
    gates = np.ones((1, L, 1))
    A_tab = np.repeat(a["A"][:, None], N, axis=1)[None]  # [E=1, D, N]
    y_ref, _, h_ref, _ = O.selective_scan(x, np.zeros_like(x), dt_mix, Bm, Cm, idx, gates, A_tab, a["D_skip"],
                                          h0=a["S0"][:, 0, :][None])
    np.testing.assert_allclose(y[:, :, 0], y_ref[0], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S[:, 0, :], h_ref[0], rtol=1e-12, atol=1e-12)


def test_identical_experts_equal_one_expert():
    a = ssd_inputs(k=3, seed=4)
    for name in ("X", "B", "C"):
        a[name] = np.repeat(a[name][:, :1], 3, axis=1)
    y3, S3 = SSD.ssd_scan_sequential(**a)
    one = dict(a, X=a["X"][:, :1], B=a["B"][:, :1], C=a["C"][:, :1], gates=np.ones((a["X"].shape[0], 1)))
    y1, S1 = SSD.ssd_scan_sequential(**one)
    np.testing.assert_allclose(y3, y1, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S3, S1, rtol=1e-12, atol=1e-12)


def test_superposition_in_X_and_the_state():
    a = ssd_inputs(seed=5)
    g = np.random.default_rng(6)
    X2 = g.standard_normal(a["X"].shape)
    S2 = g.standard_normal(a["S0"].shape)
    f = lambda X, S0: SSD.ssd_scan_sequential(**dict(a, X=X, S0=S0))
    y1, s1 = f(a["X"], a["S0"])
    y2, s2 = f(X2, S2)
    y12, s12 = f(a["X"] + 2.0 * X2, a["S0"] + 2.0 * S2)
    np.testing.assert_allclose(y12, y1 + 2.0 * y2, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(s12, s1 + 2.0 * s2, rtol=1e-11, atol=1e-11)


def test_state_decays_freely_without_input():
    a = ssd_inputs(seed=7)
    a["X"] = np.zeros_like(a["X"])
    _, S = SSD.ssd_scan_sequential(**a)
    ref = np.exp(a["delta"].sum(axis=0) * a["A"])[:, None, None] * a["S0"]
    np.testing.assert_allclose(S, ref, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("Q", [1, 3, 4, 11, 64])
def test_chunked_form_equals_sequential(Q):
    a = ssd_inputs(L=11, k=2, H=3, P=4, N=5, seed=8)
    y, S = SSD.ssd_scan_sequential(**a)
    yc, Sc = SSD.ssd_scan_chunked(**a, Q=Q)
    np.testing.assert_allclose(yc, y, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(Sc, S, rtol=1e-11, atol=1e-12)


def test_chunked_zero_state_when_absent():
    a = ssd_inputs(L=6, seed=9)
    a["S0"] = None
    y, S = SSD.ssd_scan_sequential(**a)
    yc, Sc = SSD.ssd_scan_chunked(**a, Q=4)
    np.testing.assert_allclose(yc, y, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(Sc, S, rtol=1e-11, atol=1e-12)
