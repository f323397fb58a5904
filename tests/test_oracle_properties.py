"""Property-based pins for the oracle (hypothesis): invariants that hold for every input,
checked on generated cases beyond the fixed seeds of test_oracle_pins.py."""
import math

import numpy as np
import torch
from hypothesis import given, settings
from hypothesis import strategies as st
from hypothesis.extra import numpy as hnp

from oracle import moe_oracle as O

SETTINGS = settings(max_examples=60, deadline=None)
finite32 = st.floats(min_value=-3e4, max_value=3e4, allow_nan=False, allow_infinity=False, width=32)


@SETTINGS
@given(st.integers(1, 12), st.integers(1, 6), st.booleans(), st.integers(0, 1), st.data())
def test_route_invariants(E, k, renorm, shared, data):
    k = min(k, E)
    T = data.draw(st.integers(1, 6))
    logits = data.draw(hnp.arrays(np.float32, (T, E), elements=st.floats(-8, 8, width=32)))
    ids, w = O.route(logits, k, renorm, shared)
    assert ids.shape == (T, k + shared) and w.shape == (T, k + shared)
    for t in range(T):
        sel = ids[t, :k]
        assert len(set(sel.tolist())) == k                   # distinct experts
        # no unselected expert beats a selected one; ties go to the lower index
        for e in range(E):
            if e not in sel:
                assert all(logits[t, e] < logits[t, s] or (logits[t, e] == logits[t, s] and s < e) for s in sel)
        assert np.all(w[t, :k] > 0)
        if renorm:
            assert abs(float(np.sum(w[t, :k], dtype=np.float64)) - 1.0) < 1e-5
        else:
            assert float(np.sum(w[t, :k], dtype=np.float64)) <= 1.0 + 1e-5
        if shared:
            assert ids[t, k] == E and w[t, k] == 1.0


@SETTINGS
@given(st.integers(1, 9), st.sampled_from([1, 4, 16, 128]), st.data())
def test_align_is_a_padded_stable_permutation(E, bm, data):
    P = data.draw(st.integers(0, 60))
    ids = np.array(data.draw(st.lists(st.integers(0, E - 1), min_size=P, max_size=P)), dtype=np.int32)
    a = O.align(ids, E, bm)
    s, off, p2r = a["sorted_pair_ids"], a["expert_offsets"], a["pair_to_row"]
    assert off[0] == 0 and np.all(np.diff(off) % bm == 0) and np.all(np.diff(off) >= 0)
    real = s[s < P]
    assert sorted(real.tolist()) == list(range(P))           # every pair exactly once
    for e in range(E):
        seg = s[off[e]:off[e + 1]]
        mine = seg[seg < P]
        assert np.all(ids[mine] == e) and np.all(np.diff(mine) > 0)   # own pairs, ascending
        assert np.all(seg[len(mine):] == P) and len(seg) - len(mine) < bm  # then the sentinel padding
    assert np.all(s[p2r] == np.arange(P))


@SETTINGS
@given(hnp.arrays(np.float32, st.integers(1, 64), elements=finite32))
def test_e4m3_encode_matches_torch_within_range(x):
    x = np.clip(x, -448, 448)
    want = torch.from_numpy(x.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(O.e4m3_encode(x), want)


@SETTINGS
@given(hnp.arrays(np.float32, st.tuples(st.integers(1, 3), st.sampled_from([32, 64, 96])),
                  elements=st.floats(-1e3, 1e3, width=32)))
def test_quant_mx_invariants(x):
    q, s = O.quant_mx(x)
    d = O.dequant_mx(q, s)
    blocks = x.reshape(x.shape[0], -1, 32).astype(np.float64)
    amax = np.abs(blocks).max(-1)
    e = s.astype(np.int64) - 127
    nz = amax > 0
    # the block maximum lands in [256, 512) after scaling, unless the exponent was clamped
    scaled = amax * np.ldexp(1.0, (-e).astype(np.int32))
    assert np.all((scaled[nz] >= 256) & (scaled[nz] < 512) | (e[nz] == -127))
    assert np.all(s[~nz] == 0)
    # signs survive, magnitudes never exceed 448 * 2^e, and values below it round to within half a step
    assert np.all(np.sign(d) * np.sign(x) >= 0)
    lim = np.repeat(448.0 * np.ldexp(1.0, e.astype(np.int32)), 32, 1)
    assert np.all(np.abs(d) <= lim)
    inside = np.abs(x) <= lim
    tol = np.abs(x) * 2.0 ** -4 + np.repeat(np.ldexp(1.0, e.astype(np.int32)), 32, 1) * 2.0 ** -10
    assert np.all(np.abs(d - x)[inside] <= tol[inside])


@SETTINGS
@given(hnp.arrays(np.float32, st.integers(1, 48), elements=st.floats(-10, 10, width=32)))
def test_e2m1_nearest_value(x):
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    d = O.e2m1_decode(O.e2m1_encode(x))
    a = np.minimum(np.abs(x).astype(np.float64), 6.0)
    best = np.abs(a[:, None] - grid[None, :]).min(1)
    assert np.all(np.abs(np.abs(d) - a) == best)             # a nearest grid value
    assert np.all(np.sign(d) * np.sign(x) >= 0)
