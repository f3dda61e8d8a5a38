"""Property-based pins of the oracle (CPU only, hypothesis): random
medium-size problems -- ids that may repeat inside a token or fall outside
[0, G), placement entries that may be invalid -- checked against the
pure-Python statement of the layout (``layout_defs``), and the combines
against their float64 bounds on the same random layouts."""
import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle
from layout_defs import py_layout
from test_oracle_layout import _cmp


@st.composite
def problems(draw):
    M = draw(st.integers(0, 40))
    G = draw(st.integers(1, 24))
    topk = draw(st.integers(1, 6))
    E = draw(st.integers(1, 6))
    ids = st.integers(-2, G + 1)            # a few invalid ids at both ends
    idx = draw(st.lists(st.lists(ids, min_size=topk, max_size=topk), min_size=M, max_size=M))
    po = draw(st.lists(st.integers(-1, E), min_size=G, max_size=G))
    return M, G, topk, E, idx, po, draw(st.booleans())


SETTINGS = settings(max_examples=150, deadline=None, derandomize=True,
                    suppress_health_check=[HealthCheck.too_slow])


@SETTINGS
@given(problems())
def test_layout_matches_the_definition(p):
    M, G, topk, E, idx, po, dedup = p
    idx_a = np.array(idx, np.int32).reshape(M, topk)
    o = oracle.layout(idx_a, np.array(po, np.int32), G, E, dedup)
    _cmp(o, py_layout(idx if M else [], po, G, E, dedup), dedup)


@SETTINGS
@given(problems(), st.integers(0, 2 ** 31 - 1))
def test_combines_within_float64_bounds(p, seed):
    M, G, topk, E, idx, po, _ = p
    if M == 0:
        return
    rng = np.random.default_rng(seed)
    idx_a = np.array(idx, np.int32).reshape(M, topk)
    po_a = np.array(po, np.int32)
    lay = oracle.layout(idx_a, po_a, G, E, True)
    N = 16
    R = M * topk
    y = oracle.bf16_round(rng.standard_normal((R, N)).astype(np.float32))
    w = rng.standard_normal((M, topk)).astype(np.float32)
    yf = oracle.bits_to_f32(y).astype(np.float64)
    er = lay["exp_row"]
    valid = er >= 0
    terms = np.where(valid[:, :, None], w.astype(np.float64)[:, :, None] * yf[np.where(valid, er, 0)], 0.0)
    exact, mag = terms.sum(1), np.abs(terms).sum(1)
    out = oracle.bits_to_f32(oracle.combine(y, w, er)).astype(np.float64)
    assert np.all(np.abs(out - exact) <= np.abs(exact) * 2.0 ** -8 + topk * 2.0 ** -23 * mag + 1e-37)
    z = oracle.combine_partial(y, w, idx_a, po_a, lay)
    two = oracle.bits_to_f32(oracle.combine_reduce(z, lay["disp_row"])).astype(np.float64)
    # two roundings: each partition row once (after an fp32 chain of up to
    # topk terms), the token sum once (after up to E fp32 additions)
    bound = np.abs(exact) * 2.0 ** -8 + mag * (2.0 ** -8 * (1 + 2.0 ** -8) + (topk + E) * 2.0 ** -23) + 1e-37
    assert np.all(np.abs(two - exact) <= bound)
