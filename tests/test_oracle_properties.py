"""Property-based checks of the fp64 oracle over random shapes (CPU only).

The fixed-seed pins of test_oracle_pins.py are restated here as properties that must hold for
any shape hypothesis draws:
  * reversal: the reverse scan is the forward scan of the flipped sequence ("Vision Mamba"
    sec. 2.2), bit for bit;
  * continuation: scanning [0, T) and then [T, L) from the first part's final state equals one
    scan of [0, L) (the affine recurrence of "Understanding Mamba from zero" sec. 5 carried
    across the split), to fp64 rounding;
  * superposition: a K-direction scan equals the sum of its directions' single scans, gated
    ("S4 -> Mamba" sec. 3, the SS2D merge).
"""

import numpy as np
from hypothesis import given, settings, strategies as st

import oracle

FWD, REV, COL, COLREV = 0, 1, 2, 3


def _case(seed, batch, L, D, N, K=1):
    rng = np.random.default_rng(seed)
    return dict(u=rng.standard_normal((batch, L, D)), z=rng.standard_normal((batch, L, D)),
                delta=rng.standard_normal((K, batch, L, D)),
                B=rng.standard_normal((K, batch, L, N)), C=rng.standard_normal((K, batch, L, N)),
                A=-rng.uniform(0.05, 2.0, size=(D, N)), Dskip=rng.standard_normal(D),
                delta_bias=rng.uniform(-3.0, 0.5, size=D))


def _rel(a, b):
    rms = float(np.sqrt(np.mean(b * b))) if b.size else 1.0
    return float(np.max(np.abs(a - b) / (np.abs(b) + 1e-2 * rms + 1e-300))) if b.size else 0.0


shapes = dict(seed=st.integers(0, 2 ** 31 - 1), batch=st.integers(1, 3), L=st.integers(1, 40),
              D=st.integers(1, 5), N=st.integers(1, 6))


@settings(max_examples=25, deadline=None)
@given(**shapes)
def test_reversal_is_the_flipped_forward_scan(seed, batch, L, D, N):
    c = _case(seed, batch, L, D, N)
    args = dict(Dskip=c["Dskip"], delta_bias=c["delta_bias"])
    rev, last_r = oracle.selective_scan(c["u"], c["delta"], c["A"], c["B"], c["C"], z=c["z"],
                                        dirs=(REV,), **args)
    fwd, last_f = oracle.selective_scan(c["u"][:, ::-1], c["delta"], c["A"], c["B"], c["C"],
                                        z=c["z"][:, ::-1], dirs=(FWD,), **args)
    assert np.array_equal(rev, fwd[:, ::-1]) and np.array_equal(last_r, last_f)


@settings(max_examples=25, deadline=None)
@given(split=st.floats(0.0, 1.0), **shapes)
def test_continuation_through_the_final_state(seed, batch, L, D, N, split):
    c = _case(seed, batch, L, D, N)
    T = int(round(split * L))
    args = dict(Dskip=c["Dskip"], delta_bias=c["delta_bias"])
    out, last = oracle.selective_scan(c["u"], c["delta"], c["A"], c["B"], c["C"], z=c["z"], **args)
    o1, h1 = oracle.selective_scan(c["u"][:, :T], c["delta"][:, :, :T], c["A"], c["B"][:, :, :T],
                                   c["C"][:, :, :T], z=c["z"][:, :T], **args)
    o2, h2 = oracle.selective_scan(c["u"][:, T:], c["delta"][:, :, T:], c["A"], c["B"][:, :, T:],
                                   c["C"][:, :, T:], z=c["z"][:, T:], initial_state=h1, **args)
    assert _rel(np.concatenate([o1, o2], axis=1), out) < 1e-12
    assert _rel(h2, last) < 1e-12


@settings(max_examples=20, deadline=None)
@given(seed=st.integers(0, 2 ** 31 - 1), batch=st.integers(1, 2), H=st.integers(1, 6),
       W=st.integers(1, 6), D=st.integers(1, 4), N=st.integers(1, 5),
       dirs=st.lists(st.sampled_from([FWD, REV, COL, COLREV]), min_size=1, max_size=4))
def test_directions_superpose(seed, batch, H, W, D, N, dirs):
    K = len(dirs)
    c = _case(seed, batch, H * W, D, N, K=K)
    args = dict(Dskip=c["Dskip"], delta_bias=c["delta_bias"], H=H, W=W)
    out, last = oracle.selective_scan(c["u"], c["delta"], c["A"], c["B"], c["C"], z=c["z"],
                                      dirs=tuple(dirs), **args)
    total = np.zeros_like(c["u"])
    for k, d in enumerate(dirs):
        y, l_k = oracle.selective_scan(c["u"], c["delta"][k:k + 1], c["A"], c["B"][k:k + 1],
                                       c["C"][k:k + 1], z=None, dirs=(d,), **args)
        total += y
        assert np.array_equal(l_k[0], last[k])
    gate = c["z"] / (1.0 + np.exp(-c["z"]))
    assert _rel(out, total * gate) < 1e-12
