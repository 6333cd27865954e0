"""Pins for the fp64 oracle: checks against things other than itself.

* a hand-worked example with exact fractions (tests/golden/worked_example.txt);
* a brute-force quadratic (attention-matrix) form on tiny inputs;
* closed forms: a = 1 with one frame (plain non-causal ReLU linear attention,
  evaluated in the N x N attention-matrix order), a = 0 (frame-local only),
  a = 1 over many frames (cumulative block-causal linear attention, as in the
  SANA-Video talk's block KV cache);
* chunking invariance: one call equals streaming through state_in/state_out;
* invariants: scale, permutation, linearity, convex-hull bounds;
* planted mistakes: plausible bugs in the recurrence must fail the pins.
"""

import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import gla_bruteforce_head, gla_forward, gla_head, relu, sigmoid
from workloads import WORKLOADS, make_inputs, make_state

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_example.txt")


def _rng_case(seed, F, T, d, state=True, g_mu=1.0, g_sigma=1.5):
    r = np.random.default_rng(seed)
    N = F * T
    q = r.standard_normal((N, d))
    k = r.standard_normal((N, d))
    v = r.standard_normal((N, d))
    g = r.normal(g_mu, g_sigma, F)
    s = r.standard_normal((d, d + 1)) if state else None
    if s is not None:
        s[:, d] = np.abs(s[:, d]) + 1.0  # keep the normaliser away from zero
    return q, k, v, g, s


def _parse_golden(path):
    vals = {}
    with open(path) as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, rest = line.split(":", 1)
            rows = [[Fraction(x) for x in row.split()] for row in rest.split(";")]
            vals[key.strip()] = rows
    return vals


def _as_array(rows):
    return np.array([[float(x) for x in r] for r in rows], dtype=np.float64)


# ---------------------------------------------------------------- golden


def test_golden_worked_example():
    gv = _parse_golden(GOLDEN)
    d = int(gv["d"][0][0])
    T = int(gv["T"][0][0])
    F = int(gv["F"][0][0])
    eps = float(gv["eps"][0][0])
    g = _as_array(gv["g"]).reshape(-1)
    assert g.shape == (F,)
    out, s = gla_head(_as_array(gv["q"]), _as_array(gv["k"]), _as_array(gv["v"]), g, T,
                      _as_array(gv["state_in"]), eps)
    assert out.shape == (F * T, d)
    np.testing.assert_allclose(out, _as_array(gv["out"]), rtol=0, atol=1e-15)
    np.testing.assert_allclose(s, _as_array(gv["state_out"]), rtol=0, atol=1e-15)
    # the brute-force form reaches the same hand-worked values
    out_b, s_b = gla_bruteforce_head(_as_array(gv["q"]), _as_array(gv["k"]), _as_array(gv["v"]),
                                     g, T, _as_array(gv["state_in"]), eps)
    np.testing.assert_allclose(out_b, _as_array(gv["out"]), rtol=0, atol=1e-15)
    np.testing.assert_allclose(s_b, _as_array(gv["state_out"]), rtol=0, atol=1e-15)


def test_sigmoid_special_values():
    a = sigmoid(np.array([-np.inf, 0.0, np.inf]))
    assert a[0] == 0.0 and a[1] == 0.5 and a[2] == 1.0


def test_relu_signed_zero():
    z = relu(np.array([-0.0, -1.0, 2.0]))
    assert np.signbit(z).tolist() == [False, False, False]
    assert z.tolist() == [0.0, 0.0, 2.0]


# ----------------------------------------------------------- brute force


@pytest.mark.parametrize(
    "seed,F,T,d,state",
    [(1, 4, 16, 32, False), (2, 2, 37, 32, True), (3, 3, 5, 64, True),
     (4, 1, 9, 8, True), (5, 5, 3, 16, False), (6, 2, 1, 4, True)],
)
def test_bruteforce_matches_oracle(seed, F, T, d, state):
    q, k, v, g, s = _rng_case(seed, F, T, d, state)
    out, so = gla_head(q, k, v, g, T, s)
    out_b, so_b = gla_bruteforce_head(q, k, v, g, T, s)
    np.testing.assert_allclose(out, out_b, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(so, so_b, rtol=1e-10, atol=1e-10)


def test_bruteforce_tiny_workload():
    """The tiny workload exactly as the library receives it (bf16 inputs)."""
    w = WORKLOADS["tiny"]
    q, k, v, g = make_inputs(w)
    out, so = gla_forward(q, k, v, g, w.frames, None, w.eps)
    for b in range(w.B):
        for h in range(w.H):
            ob, sb = gla_bruteforce_head(q[b, :, h], k[b, :, h], v[b, :, h], g[b, :, h],
                                         w.tokens_per_frame, None, w.eps)
            np.testing.assert_allclose(out[b, :, h], ob, rtol=1e-10, atol=1e-12)
            np.testing.assert_allclose(so[b, h], sb, rtol=1e-10, atol=1e-10)


def test_bruteforce_gate_extremes():
    q, k, v, _, s = _rng_case(7, 4, 6, 8, True)
    g = np.array([np.inf, -np.inf, 0.3, np.inf])
    out, so = gla_head(q, k, v, g, 6, s)
    ob, sb = gla_bruteforce_head(q, k, v, g, 6, s)
    np.testing.assert_allclose(out, ob, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(so, sb, rtol=1e-10, atol=1e-10)


# ----------------------------------------------------------- closed forms


def _attention_matrix_form(q, k, v, mask, eps):
    """Textbook linear attention in N x N order: A = phi(Q) phi(K)^T (masked),
    out = A V / (A 1 + eps)."""
    A = np.maximum(q, 0) @ np.maximum(k, 0).T
    A = A * mask
    return (A @ v) / (A.sum(axis=1) + eps)[:, None]


def test_closed_form_a1_single_frame():
    """a = 1, one frame, zero state: plain non-causal ReLU linear attention."""
    q, k, v, _, _ = _rng_case(11, 1, 50, 16, False)
    out, so = gla_head(q, k, v, np.array([np.inf]), 50, None, 1e-6)
    ref = _attention_matrix_form(q, k, v, np.ones((50, 50)), 1e-6)
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-13)
    # the state is the single frame's increment phi(K)^T [V | 1]
    pk = np.maximum(k, 0)
    np.testing.assert_allclose(so[:, :16], pk.T @ v, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(so[:, 16], pk.sum(axis=0), rtol=1e-12, atol=1e-12)


def test_closed_form_a0_frame_local():
    """a = 0: every frame sees only itself and state_in is erased."""
    F, T, d = 4, 12, 16
    q, k, v, _, s = _rng_case(12, F, T, d, True)
    g = np.full(F, -np.inf)
    out, so = gla_head(q, k, v, g, T, s, 1e-6)
    for f in range(F):
        rows = slice(f * T, (f + 1) * T)
        ref = _attention_matrix_form(q[rows], k[rows], v[rows], np.ones((T, T)), 1e-6)
        np.testing.assert_allclose(out[rows], ref, rtol=1e-11, atol=1e-13)
    last = slice((F - 1) * T, F * T)
    pk = np.maximum(k[last], 0)
    np.testing.assert_allclose(so[:, :d], pk.T @ v[last], rtol=1e-12, atol=1e-12)
    # a different state_in changes nothing
    out2, so2 = gla_head(q, k, v, g, T, 5.0 * s, 1e-6)
    np.testing.assert_array_equal(out, out2)
    np.testing.assert_array_equal(so, so2)


def test_closed_form_a1_many_frames_block_causal():
    """a = 1 over many frames: cumulative block-causal linear attention
    (queries of frame f see the keys of frames 0..f)."""
    F, T, d = 5, 7, 8
    q, k, v, _, _ = _rng_case(13, F, T, d, False)
    fr = np.arange(F * T) // T
    mask = (fr[None, :] <= fr[:, None]).astype(np.float64)
    out, _ = gla_head(q, k, v, np.full(F, np.inf), T, None, 1e-6)
    ref = _attention_matrix_form(q, k, v, mask, 1e-6)
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-13)


# ------------------------------------------------------ chunking invariance


@pytest.mark.parametrize("splits", [[1, 1, 1, 1, 1, 1], [2, 4], [5, 1], [3, 3], [6]])
def test_chunking_invariance(splits):
    F, T, d = 6, 9, 16
    q, k, v, g, s = _rng_case(21, F, T, d, True, g_mu=2.0, g_sigma=1.0)
    out_all, s_all = gla_head(q, k, v, g, T, s)
    state = s
    f0 = 0
    outs = []
    for n in splits:
        rows = slice(f0 * T, (f0 + n) * T)
        o, state = gla_head(q[rows], k[rows], v[rows], g[f0:f0 + n], T, state)
        outs.append(o)
        f0 += n
    np.testing.assert_allclose(np.vstack(outs), out_all, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(state, s_all, rtol=1e-12, atol=1e-12)


def test_batched_equals_per_head():
    w = WORKLOADS["tiny"].with_(B=2, H=3, random_state_in=True)
    q, k, v, g = make_inputs(w, seed=99)
    s = make_state(w, seed=99)
    out, so = gla_forward(q, k, v, g, w.frames, s, w.eps)
    for b in range(2):
        for h in range(3):
            o, st = gla_head(q[b, :, h], k[b, :, h], v[b, :, h], g[b, :, h], w.tokens_per_frame,
                             s[b, h], w.eps)
            np.testing.assert_array_equal(out[b, :, h], o)
            np.testing.assert_array_equal(so[b, h], st)


# ---------------------------------------------------------------- invariants


def test_query_scale_invariance():
    q, k, v, g, s = _rng_case(31, 3, 10, 8, True)
    o1, _ = gla_head(q, k, v, g, 10, s, 0.0)
    o2, _ = gla_head(4.0 * q, k, v, g, 10, s, 0.0)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-14)


def test_key_scale_invariance_zero_state():
    q, k, v, g, _ = _rng_case(32, 3, 10, 8, False)
    o1, _ = gla_head(q, k, v, g, 10, None, 0.0)
    o2, _ = gla_head(q, 0.125 * k, v, g, 10, None, 0.0)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-14)


def test_permutation_within_frame():
    F, T, d = 3, 8, 8
    q, k, v, g, s = _rng_case(33, F, T, d, True)
    o, so = gla_head(q, k, v, g, T, s)
    r = np.random.default_rng(0)
    perm = np.concatenate([f * T + r.permutation(T) for f in range(F)])
    # permuting queries permutes outputs; permuting keys/values changes nothing
    oq, _ = gla_head(q[perm], k, v, g, T, s)
    np.testing.assert_allclose(oq, o[perm], rtol=1e-12, atol=1e-14)
    okv, sokv = gla_head(q, k[perm], v[perm], g, T, s)
    np.testing.assert_allclose(okv, o, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(sokv, so, rtol=1e-12, atol=1e-12)


def test_linearity_in_v_and_convex_hull():
    F, T, d = 3, 10, 8
    q, k, v1, g, _ = _rng_case(34, F, T, d, False)
    v2 = np.random.default_rng(5).standard_normal(v1.shape)
    o1, _ = gla_head(q, k, v1, g, T)
    o2, _ = gla_head(q, k, v2, g, T)
    o12, _ = gla_head(q, k, 2.0 * v1 - 3.0 * v2, g, T)
    np.testing.assert_allclose(o12, 2.0 * o1 - 3.0 * o2, rtol=1e-10, atol=1e-12)
    # with zero state the output is a sub-convex combination of seen values and 0
    lo = np.minimum(0.0, v1.min(axis=0))
    hi = np.maximum(0.0, v1.max(axis=0))
    assert np.all(o1 >= lo - 1e-12) and np.all(o1 <= hi + 1e-12)
    # constant values: out = c * den / (den + eps)
    c = np.linspace(-1, 1, d)
    oc, sc = gla_head(q, k, np.tile(c, (F * T, 1)), g, T, None, 0.0)
    mask = relu(q).sum(axis=1) > 0
    np.testing.assert_allclose(oc[mask], np.tile(c, (mask.sum(), 1)), rtol=1e-12, atol=1e-13)


def test_state_size_independent_of_length():
    for F, T in [(1, 1), (2, 50), (7, 3)]:
        q, k, v, g, _ = _rng_case(40 + F, F, T, 8, False)
        _, so = gla_head(q, k, v, g, T)
        assert so.shape == (8, 9)


def test_empty_cases():
    d = 8
    s = np.random.default_rng(1).standard_normal((d, d + 1))
    # no frames: state passes through unchanged
    o, so = gla_head(np.zeros((0, d)), np.zeros((0, d)), np.zeros((0, d)), np.zeros(0), 0, s)
    assert o.shape == (0, d)
    np.testing.assert_array_equal(so, s)
    # frames with no tokens: only the decay acts
    g = np.array([0.0, 1.0, -2.0])
    o, so = gla_head(np.zeros((0, d)), np.zeros((0, d)), np.zeros((0, d)), g, 0, s)
    a = sigmoid(g)
    np.testing.assert_allclose(so, a[0] * a[1] * a[2] * s, rtol=1e-15)


# -------------------------------------------------------- planted mistakes


def _mutant(kind):
    """The oracle's recurrence with one plausible mistake planted."""

    @np.errstate(divide="ignore", invalid="ignore")
    def run(q, k, v, g, T, s_in=None, eps=1e-6):
        q, k, v, g = (np.asarray(x, np.float64) for x in (q, k, v, g))
        F, d = g.shape[0], q.shape[1]
        S = np.zeros((d, d + 1)) if s_in is None else np.array(s_in, np.float64)
        out = np.zeros((F * T, d))
        a = 1.0 / (1.0 + np.exp(-g))
        if kind == "one_minus_a":
            a = 1.0 - a
        for f in range(F):
            r = slice(f * T, (f + 1) * T)
            K = np.maximum(k[r], 0)
            V = v[r] if kind != "relu_on_v" else np.maximum(v[r], 0)
            dS = K.T @ np.hstack([V, np.ones((T, 1))])
            if kind == "transposed_increment":
                dS = np.hstack([dS[:, :d].T, dS[:, d:]])
            S_prev = S
            S = a[f] * (S + dS) if kind == "decay_after_add" else a[f] * S + dS
            Sread = S_prev if kind == "read_previous_state" else S
            Q = np.maximum(q[r], 0) if kind != "no_relu_on_q" else q[r]
            den = Q @ Sread[:, d]
            if kind == "den_from_wrong_column":
                den = Q @ Sread[:, d - 1]
            out[r] = (Q @ Sread[:, :d]) / (den + eps)[:, None]
        return out, S

    return run


@pytest.mark.parametrize("kind", ["one_minus_a", "relu_on_v", "transposed_increment",
                                  "decay_after_add", "read_previous_state", "no_relu_on_q",
                                  "den_from_wrong_column"])
def test_planted_mistakes_fail_the_pins(kind):
    """Each planted mistake must be caught by the brute-force pin or the
    hand-worked example; the unmodified recurrence passes both."""
    q, k, v, g, s = _rng_case(50, 4, 6, 8, True)
    ob, sb = gla_bruteforce_head(q, k, v, g, 6, s)
    om, sm = _mutant(kind)(q, k, v, g, 6, s)
    err_brute = max(np.abs(om - ob).max() / np.abs(ob).max(),
                    np.abs(sm - sb).max() / np.abs(sb).max())
    gv = _parse_golden(GOLDEN)
    og, sg = _mutant(kind)(_as_array(gv["q"]), _as_array(gv["k"]), _as_array(gv["v"]),
                           _as_array(gv["g"]).reshape(-1), 2, _as_array(gv["state_in"]), 0.0)
    err_gold = max(np.abs(og - _as_array(gv["out"])).max(),
                   np.abs(sg - _as_array(gv["state_out"])).max())
    err_brute, err_gold = np.nan_to_num([err_brute, err_gold], nan=np.inf)
    assert max(err_brute, err_gold) > 1e-3, kind
    # control: the same harness with no mistake planted agrees
    oc, sc = _mutant("none")(q, k, v, g, 6, s)
    np.testing.assert_allclose(oc, ob, rtol=1e-10, atol=1e-12)


def test_torch_bf16_inputs_widen_exactly():
    x = torch.tensor([1.0, -2.5, 3.140625], dtype=torch.bfloat16)
    y = relu(x)
    assert y.dtype == np.float64 and y.tolist() == [1.0, 0.0, 3.140625]
