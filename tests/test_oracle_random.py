"""Randomised pins of the fp64 oracle on tiny shapes (CPU only): the forward
against pure-Python softmax loops, the backward against central finite
differences, over random head groupings, unequal query / key lengths, causal
on and off, and random scales.  The fixed-shape versions of the same pins
live in test_oracle.py; these draw the shapes as well (from a fixed
example sequence, so every run checks the same cases)."""
import math

import numpy as np
from hypothesis import given, settings, strategies as st

import oracle
from tests.test_oracle import brute_force, finite_difference_grads, rel_err

shapes = st.fixed_dictionaries({
    "B": st.integers(1, 2),
    "Hkv": st.integers(1, 2),
    "g": st.integers(1, 3),
    "Nq": st.integers(1, 9),
    "Nk": st.integers(1, 9),
    "d": st.integers(1, 6),
    "causal": st.booleans(),
    "scale": st.floats(0.1, 1.5),
    "seed": st.integers(0, 2**31 - 1),
})


def draw(s, with_do=False):
    rng = np.random.default_rng(s["seed"])
    Hq = s["Hkv"] * s["g"]
    q = rng.standard_normal((s["B"], Hq, s["Nq"], s["d"]))
    k = rng.standard_normal((s["B"], s["Hkv"], s["Nk"], s["d"]))
    v = rng.standard_normal((s["B"], s["Hkv"], s["Nk"], s["d"]))
    do = rng.standard_normal(q.shape) if with_do else None
    return q, k, v, do


@settings(max_examples=40, deadline=None, derandomize=True)
@given(shapes)
def test_forward_matches_python_loops(s):
    q, k, v, _ = draw(s)
    o, lse = oracle.attention_forward(q, k, v, s["causal"], s["scale"])
    ob, lb = brute_force(q.tolist(), k.tolist(), v.tolist(), s["causal"], s["scale"])
    np.testing.assert_allclose(o, np.array(ob), atol=1e-12, rtol=1e-12)
    np.testing.assert_allclose(lse, np.array(lb), atol=1e-12, rtol=1e-12)


@settings(max_examples=8, deadline=None, derandomize=True)
@given(shapes.filter(lambda s: s["B"] * s["Hkv"] * s["g"] * max(s["Nq"], s["Nk"]) * s["d"] <= 120))
def test_backward_matches_finite_differences(s):
    q, k, v, do = draw(s, with_do=True)
    got = oracle.attention_backward(q, k, v, do, s["causal"], s["scale"])
    ref = finite_difference_grads(q, k, v, do, s["causal"], s["scale"])
    for g, r in zip(got, ref):
        assert rel_err(g, r) < 1e-6 or float(np.abs(r).max()) < 1e-9
        assert math.isfinite(float(np.abs(g).max()))
