"""Pins of the fp64 oracle to facts the pages and the mathematics fix (CPU only).

The pages print no numerical worked example for this path, so every pin is a closed form, an
identity, a special case or a brute force that does not run the oracle's recurrence loop:

  P1  constant Delta, B, C (an LTI system): the output is the convolution y = u * K with
      K_j = sum_n C_n Abar_n^j Bbar_n ("Understanding Mamba from zero" sec. 2.3, eq. 3),
      Abar^j taken in closed form exp(j*Delta*A), never iterated.  Checked for the Delta*B
      reading and for eq. 4's exact ZOH Bbar.
  P2  Delta = 0 leaves the state unchanged (Abar = 1, Bbar = 0): a step with Delta = 0 reads
      out C_t . h_{t-1}, and deleting such steps leaves last_state bit-identical; with softplus
      on, Delta -> 0 as delta_raw -> -inf.
  P3  the reverse scan equals the forward scan of the flipped sequence (Vim backward scan,
      "Vision Mamba" sec. 2.2).
  P4  SS2D (four cross-scan orders, "S4 -> Mamba" sec. 3) and Vim (two orders) equal single
      forward scans of explicitly permuted tensors (permutations written as (i, j) double loops),
      inverse-permuted and summed, then gated.
  P5  Theorem 1 (sec. 6.2 Step 5): with N = 1, A = -1, B = C = 1, softplus on, the scan is the
      gated recurrence h_t = (1 - g_t) h_{t-1} + w_t u_t with g_t = sigmoid(r_t); w_t = g_t for
      eq. 4's exact ZOH and w_t = softplus(r_t) for Bbar = Delta*B.
  P6  unrolled double sum: y_t = sum_{s<=t} sum_n C_t[n] exp(A_n sum_{r=s+1..t} Delta_r)
      Delta_s B_s[n] u_s + D u_t, brute force in O(L^2 N).
  P7  chunk associativity of the affine recurrence (sec. 5; "S4 -> Mamba" sec. 2.2): splitting
      the sequence at T, the end state is exp(A * sum Delta_suffix) * h_prefix + h_suffix(0), and
      the suffix outputs gain C_t . (exp(A * partial sums) * h_prefix).
  P8  linearity in u with no gate, and the decay bound |h_n| <= sum_s |Delta_s B_s[n] u_s|.
  P9  the causal depthwise convolution + SiLU before the scan ("Understanding Mamba from zero"
      sec. 6.2 Step 2; "Vision Mamba" sec. 2.2, one convolution per scanned sequence) equals
      numpy's full convolution of each direction's explicitly permuted sequence, truncated to
      the causal part.
  P10 a scan with the convolution equals, direction by direction, single scans of the
      convolved inputs (computed as in P9, put back in spatial order), summed and gated: the
      convolved value replaces u in both the Bbar*u term and the D skip.
  P11 with an input per direction, a K-direction scan equals the sum of K single-direction
      scans of those inputs, gated; and Sigma's CroMB ("S4 -> Mamba" sec. 4.1) written as the
      pages give it, SSM(x_rgb, C=C_depth) + SSM(x_depth, C=C_rgb) from two separate scans,
      equals the two-direction scan with the C tensors stacked in swapped order.
  P13 parameters per direction: a K-direction scan whose directions carry their own A, Dskip and
      delta_bias equals the sum of K single-direction scans, each with its own parameters, gated.
  P12 int8 Delta ("S4 -> Mamba" sec. 2.3): codes q with one scale per channel scan exactly like
      the raw values q * scale[d] given directly (the products are exact in float64).
  plus the silu gate against sigmoid written out, a hand-worked Abar = 1/2 example, empty and
  length-1 inputs, and a regression fixture written by tests/golden/make_golden.py.
"""

import json
import os

import numpy as np
import pytest

import oracle
from selective_state_space_13_b200 import workloads as wl

FWD, REV, COL, COLREV = 0, 1, 2, 3
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rel_err(got, ref):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    if ref.size == 0:
        return 0.0
    rms = np.sqrt(np.mean(ref * ref))
    return float(np.max(np.abs(got - ref) / (np.abs(ref) + 1e-2 * rms + 1e-300)))


def np_softplus(x):
    return np.logaddexp(0.0, x)


def rand_case(rng, batch=2, L=23, D=3, N=4, K=1, distinct_A=True):
    u = rng.standard_normal((batch, L, D))
    z = rng.standard_normal((batch, L, D))
    delta = rng.standard_normal((K, batch, L, D))
    B = rng.standard_normal((K, batch, L, N))
    C = rng.standard_normal((K, batch, L, N))
    if distinct_A:
        A = -rng.uniform(0.1, 2.0, size=(D, N))
    else:
        A = np.tile(-(np.arange(N) + 1.0), (D, 1))
    Dskip = rng.standard_normal(D)
    bias = rng.uniform(-2.0, 0.5, size=D)
    return dict(u=u, z=z, delta=delta, B=B, C=C, A=A, Dskip=Dskip, delta_bias=bias)


# ----------------------------------------------------------------------------- P1

@pytest.mark.parametrize("zoh", [False, True])
def test_P1_lti_equals_convolution(zoh):
    rng = np.random.default_rng(1)
    batch, L, D, N = 2, 40, 3, 4
    c = rand_case(rng, batch, L, D, N)
    dt = rng.uniform(0.05, 0.6, size=D)                 # constant step per channel
    Bc = rng.standard_normal((batch, N))
    Cc = rng.standard_normal((batch, N))
    delta = np.broadcast_to(dt, (1, batch, L, D)).copy()
    B = np.broadcast_to(Bc[None, :, None, :], (1, batch, L, N)).copy()
    C = np.broadcast_to(Cc[None, :, None, :], (1, batch, L, N)).copy()
    out, last = oracle.selective_scan(c["u"], delta, c["A"], B, C, Dskip=c["Dskip"], z=None,
                                      delta_bias=None, softplus=False, zoh_exact=zoh)
    ref = np.zeros((batch, L, D))
    for b in range(batch):
        for d in range(D):
            a = c["A"][d]
            bbar = (np.expm1(dt[d] * a) / a) * Bc[b] if zoh else dt[d] * Bc[b]
            kern = np.array([np.sum(Cc[b] * np.exp(j * dt[d] * a) * bbar) for j in range(L)])
            for t in range(L):
                ref[b, t, d] = sum(kern[t - s] * c["u"][b, s, d] for s in range(t + 1)) \
                    + c["Dskip"][d] * c["u"][b, t, d]
    assert rel_err(out, ref) < 1e-12


# ----------------------------------------------------------------------------- P2

def test_P2_zero_delta_steps_hold_state():
    rng = np.random.default_rng(2)
    batch, L, D, N = 2, 30, 3, 4
    c = rand_case(rng, batch, L, D, N)
    zero_steps = [0, 7, 8, 19, 29]
    delta = rng.uniform(0.01, 0.5, size=(1, batch, L, D))
    for t in zero_steps:
        delta[:, :, t, :] = -c["delta_bias"]           # delta_raw + bias == 0 exactly
    args = dict(Dskip=c["Dskip"], z=None, delta_bias=c["delta_bias"], softplus=False)
    out, last = oracle.selective_scan(c["u"], delta, c["A"], c["B"][:1], c["C"][:1], **args)
    for t in zero_steps:
        if t == 0:
            h_prev = np.zeros((1, batch, D, N))
        else:
            _, h_prev = oracle.selective_scan(c["u"][:, :t], delta[:, :, :t], c["A"],
                                              c["B"][:1, :, :t], c["C"][:1, :, :t], **args)
        y_expect = np.einsum("bn,bdn->bd", c["C"][0, :, t], h_prev[0]) + c["Dskip"] * c["u"][:, t]
        assert np.allclose(out[:, t], y_expect, rtol=1e-13, atol=1e-13)
    keep = [t for t in range(L) if t not in zero_steps]
    _, last_kept = oracle.selective_scan(c["u"][:, keep], delta[:, :, keep], c["A"],
                                         c["B"][:1, :, keep], c["C"][:1, :, keep], **args)
    assert np.array_equal(last, last_kept)


def test_P2_softplus_delta_to_zero_converges():
    rng = np.random.default_rng(3)
    batch, L, D, N = 1, 12, 2, 3
    c = rand_case(rng, batch, L, D, N)
    base = rng.standard_normal((1, batch, L, D))
    args = dict(Dskip=c["Dskip"], z=None, delta_bias=None, softplus=True)
    _, last_without = oracle.selective_scan(c["u"][:, :-1], base[:, :, :-1], c["A"],
                                            c["B"][:1, :, :-1], c["C"][:1, :, :-1], **args)
    prev = None
    for x in (-5.0, -10.0, -20.0, -40.0):
        delta = base.copy()
        delta[:, :, -1, :] = x
        _, last = oracle.selective_scan(c["u"], delta, c["A"], c["B"][:1], c["C"][:1], **args)
        gap = np.max(np.abs(last - last_without))
        assert gap <= 500.0 * np.exp(x) + 1e-15
        if prev is not None:
            assert gap <= prev
        prev = gap


# ----------------------------------------------------------------------------- P3

def test_P3_reverse_equals_flipped_forward():
    rng = np.random.default_rng(4)
    c = rand_case(rng, 2, 37, 5, 4)
    args = dict(Dskip=c["Dskip"], delta_bias=c["delta_bias"], softplus=True)
    out_r, last_r = oracle.selective_scan(c["u"], c["delta"], c["A"], c["B"], c["C"], z=c["z"],
                                          dirs=(REV,), **args)
    out_f, last_f = oracle.selective_scan(c["u"][:, ::-1], c["delta"], c["A"], c["B"], c["C"],
                                          z=c["z"][:, ::-1], dirs=(FWD,), **args)
    assert np.array_equal(out_r, out_f[:, ::-1])
    assert np.array_equal(last_r, last_f)


# ----------------------------------------------------------------------------- P4

def _perm_by_loops(kind, H, W):
    """Spatial position for every scan step, written as explicit (i, j) loops over the image."""
    L = H * W
    order = []
    if kind in (FWD, REV):
        for i in range(H):
            for j in range(W):
                order.append(i * W + j)
    else:
        for j in range(W):
            for i in range(H):
                order.append(i * W + j)
    order = np.array(order)
    if kind in (REV, COLREV):
        order = order[::-1]
    assert sorted(order.tolist()) == list(range(L))
    return order


@pytest.mark.parametrize("dirs,H,W", [((FWD, COL, REV, COLREV), 5, 7),
                                      ((FWD, REV), 1, 29),
                                      ((COL,), 6, 4),
                                      ((COLREV, FWD), 3, 3)])
def test_P4_multi_direction_equals_permuted_scans(dirs, H, W):
    rng = np.random.default_rng(5 + len(dirs))
    L = H * W
    K = len(dirs)
    c = rand_case(rng, 2, L, 3, 4, K=K)
    args = dict(Dskip=c["Dskip"], delta_bias=c["delta_bias"], softplus=True)
    out, last = oracle.selective_scan(c["u"], c["delta"], c["A"], c["B"], c["C"], z=c["z"],
                                      dirs=dirs, H=H, W=W, **args)
    total = np.zeros_like(c["u"])
    lasts = []
    for k, kind in enumerate(dirs):
        order = _perm_by_loops(kind, H, W)
        u_perm = c["u"][:, order]                       # u_perm[t] = u[position of step t]
        y_perm, l_k = oracle.selective_scan(u_perm, c["delta"][k:k + 1], c["A"], c["B"][k:k + 1],
                                            c["C"][k:k + 1], z=None, dirs=(FWD,), **args)
        y = np.empty_like(y_perm)
        y[:, order] = y_perm                            # back to spatial order
        total += y
        lasts.append(l_k[0])
    gate = c["z"] / (1.0 + np.exp(-c["z"]))
    assert rel_err(out, total * gate) < 1e-13
    assert np.array_equal(last, np.stack(lasts))


def test_oracle_position_matches_loops():
    for H, W in [(5, 7), (56, 56), (1, 9), (9, 1)]:
        L = H * W
        for kind in (FWD, REV, COL, COLREV):
            order = _perm_by_loops(kind, H, W)
            got = [oracle.position(kind, L, t, H, W) for t in range(L)]
            assert got == order.tolist()
    assert oracle.position(7, 10, 0) == -1


# ----------------------------------------------------------------------------- P5

@pytest.mark.parametrize("zoh", [False, True])
def test_P5_theorem1_gated_rnn(zoh):
    rng = np.random.default_rng(6)
    batch, L = 3, 50
    u = rng.standard_normal((batch, L, 1))
    r = 2.0 * rng.standard_normal((1, batch, L, 1))
    ones = np.ones((1, batch, L, 1))
    out, last = oracle.selective_scan(u, r, -np.ones((1, 1)), ones, ones, Dskip=np.zeros(1),
                                      z=None, delta_bias=np.zeros(1), softplus=True,
                                      zoh_exact=zoh)
    g = 1.0 / (1.0 + np.exp(-r[0, :, :, 0]))
    w = g if zoh else np.log1p(np.exp(r[0, :, :, 0]))
    h = np.zeros(batch)
    ref = np.zeros((batch, L))
    for t in range(L):
        h = (1.0 - g[:, t]) * h + w[:, t] * u[:, t, 0]
        ref[:, t] = h
    assert rel_err(out[:, :, 0], ref) < 1e-12
    assert rel_err(last[0, :, 0, 0], h) < 1e-12


# ----------------------------------------------------------------------------- P6

@pytest.mark.parametrize("distinct_A", [True, False])
def test_P6_unrolled_double_sum(distinct_A):
    rng = np.random.default_rng(7)
    batch, L, D, N = 2, 26, 3, 5
    c = rand_case(rng, batch, L, D, N, distinct_A=distinct_A)
    out, last = oracle.selective_scan(c["u"], c["delta"], c["A"], c["B"], c["C"], Dskip=c["Dskip"],
                                      z=None, delta_bias=c["delta_bias"], softplus=True)
    dlt = np_softplus(c["delta"][0] + c["delta_bias"])            # [batch, L, D]
    ref = np.zeros((batch, L, D))
    href = np.zeros((batch, D, N))
    for b in range(batch):
        for d in range(D):
            cum = np.concatenate([[0.0], np.cumsum(dlt[b, :, d])])  # cum[t+1] = sum_{r<=t}
            for t in range(L):
                acc = 0.0
                for s in range(t + 1):
                    decay = np.exp(c["A"][d] * (cum[t + 1] - cum[s + 1]))
                    acc += np.sum(c["C"][0, b, t] * decay * dlt[b, s, d] * c["B"][0, b, s]) \
                        * c["u"][b, s, d]
                ref[b, t, d] = acc + c["Dskip"][d] * c["u"][b, t, d]
            for s in range(L):
                href[b, d] += np.exp(c["A"][d] * (cum[L] - cum[s + 1])) * dlt[b, s, d] \
                    * c["B"][0, b, s] * c["u"][b, s, d]
    assert rel_err(out, ref) < 1e-11
    assert rel_err(last[0], href) < 1e-11


# ----------------------------------------------------------------------------- P7

def test_P7_chunk_carry_combine():
    rng = np.random.default_rng(8)
    batch, L, D, N, T = 2, 41, 4, 6, 17
    c = rand_case(rng, batch, L, D, N)
    args = dict(Dskip=c["Dskip"], z=None, delta_bias=c["delta_bias"], softplus=True)
    out, last = oracle.selective_scan(c["u"], c["delta"], c["A"], c["B"], c["C"], **args)
    _, h1 = oracle.selective_scan(c["u"][:, :T], c["delta"][:, :, :T], c["A"], c["B"][:, :, :T],
                                  c["C"][:, :, :T], **args)
    out2, h2 = oracle.selective_scan(c["u"][:, T:], c["delta"][:, :, T:], c["A"],
                                     c["B"][:, :, T:], c["C"][:, :, T:], **args)
    dlt = np_softplus(c["delta"][0] + c["delta_bias"])           # [batch, L, D]
    csum = np.cumsum(dlt[:, T:], axis=1)                          # partial sums over the suffix
    P = np.exp(c["A"][None] * csum[:, -1, :, None])              # [batch, D, N]
    assert rel_err(last[0], P * h1[0] + h2[0]) < 1e-12
    decay = np.exp(c["A"][None, None] * csum[..., None])         # [batch, L-T, D, N]
    corr = np.einsum("btn,btdn,bdn->btd", c["C"][0, :, T:], decay, h1[0])
    assert rel_err(out[:, T:], out2 + corr) < 1e-12


# ----------------------------------------------------------------------------- P8

def test_P8_linearity_and_decay_bound():
    rng = np.random.default_rng(9)
    c = rand_case(rng, 2, 33, 3, 4)
    args = dict(Dskip=c["Dskip"], z=None, delta_bias=c["delta_bias"], softplus=True)
    u2 = rng.standard_normal(c["u"].shape)
    o1, l1 = oracle.selective_scan(c["u"], c["delta"], c["A"], c["B"], c["C"], **args)
    o2, l2 = oracle.selective_scan(u2, c["delta"], c["A"], c["B"], c["C"], **args)
    o3, l3 = oracle.selective_scan(2.5 * c["u"] - 0.75 * u2, c["delta"], c["A"], c["B"], c["C"],
                                   **args)
    assert rel_err(o3, 2.5 * o1 - 0.75 * o2) < 1e-12
    assert rel_err(l3, 2.5 * l1 - 0.75 * l2) < 1e-12
    dlt = np_softplus(c["delta"][0] + c["delta_bias"])
    bound = np.einsum("btd,btn,btd->bdn", dlt, np.abs(c["B"][0]), np.abs(c["u"]))
    assert np.all(np.abs(l1[0]) <= bound * (1 + 1e-12))


# ----------------------------------------------------------------------------- gate, worked example, edges

def test_gate_is_silu():
    rng = np.random.default_rng(10)
    c = rand_case(rng, 1, 19, 4, 3)
    args = dict(Dskip=c["Dskip"], delta_bias=c["delta_bias"], softplus=True)
    og, _ = oracle.selective_scan(c["u"], c["delta"], c["A"], c["B"], c["C"], z=c["z"], **args)
    on, _ = oracle.selective_scan(c["u"], c["delta"], c["A"], c["B"], c["C"], z=None, **args)
    sig = 1.0 / (1.0 + np.exp(-c["z"]))
    assert rel_err(og, on * c["z"] * sig) < 1e-14


def test_hand_worked_half_decay():
    # softplus off, Delta = 1, A = -ln 2 -> Abar = exp(-ln 2) = 1/2; B = C = 1; N = 1; D = 1/2.
    # h_1 = 1, h_2 = 1/2 + 2 = 5/2, h_3 = 5/4 + 3 = 17/4, h_4 = 17/8 + 4 = 49/8 (eq. 2a);
    # y_t = h_t + u_t/2 (eq. 2b plus the skip): 3/2, 7/2, 23/4, 65/8.
    u = np.array([1.0, 2.0, 3.0, 4.0]).reshape(1, 4, 1)
    one = np.ones((1, 1, 4, 1))
    out, last = oracle.selective_scan(u, one, np.array([[-np.log(2.0)]]), one, one,
                                      Dskip=np.array([0.5]), z=None, softplus=False)
    assert np.allclose(out.ravel(), [1.5, 3.5, 5.75, 8.125], rtol=1e-15, atol=0)
    assert np.isclose(last.ravel()[0], 49.0 / 8.0, rtol=1e-15, atol=0)


def test_empty_and_length_one():
    rng = np.random.default_rng(11)
    c = rand_case(rng, 2, 1, 3, 4)
    out, last = oracle.selective_scan(c["u"], c["delta"], c["A"], c["B"], c["C"], Dskip=c["Dskip"],
                                      z=None, delta_bias=c["delta_bias"], softplus=True)
    dlt = np_softplus(c["delta"][0, :, 0] + c["delta_bias"])      # [batch, D]
    h = dlt[..., None] * c["B"][0, :, 0][:, None, :] * c["u"][:, 0][..., None]
    assert rel_err(last[0], h) < 1e-14
    y = np.einsum("bn,bdn->bd", c["C"][0, :, 0], h) + c["Dskip"] * c["u"][:, 0]
    assert rel_err(out[:, 0], y) < 1e-14
    e = np.zeros((2, 0, 3))
    out, last = oracle.selective_scan(e, np.zeros((1, 2, 0, 3)), c["A"], np.zeros((1, 2, 0, 4)),
                                      np.zeros((1, 2, 0, 4)))
    assert out.shape == (2, 0, 3) and np.all(last == 0)


def test_bad_arguments_rejected():
    rng = np.random.default_rng(12)
    c = rand_case(rng, 1, 6, 2, 2)
    with pytest.raises(ValueError):
        oracle.selective_scan(c["u"], c["delta"], c["A"], c["B"], c["C"], dirs=(COL,), H=2, W=2)
    with pytest.raises(ValueError):
        oracle.selective_scan(c["u"], c["delta"], c["A"], c["B"], c["C"], dirs=(5,))


def test_golden_regression_fixture():
    path = os.path.join(GOLDEN, "tiny_oracle.json")
    with open(path) as f:
        g = json.load(f)
    inp = wl.make_inputs("tiny")
    f64 = wl.inputs_f64(inp)
    out, last = oracle.selective_scan(f64["u"], f64["delta"], f64["A"], f64["B"], f64["C"],
                                      Dskip=f64["Dskip"], z=f64["z"], delta_bias=f64["delta_bias"],
                                      softplus=True)
    assert rel_err(out, np.array(g["out"])) < 1e-13
    assert rel_err(last, np.array(g["last_state"])) < 1e-13
    # the stored inputs' checksum guards the seeded generator as well
    assert abs(float(np.sum(f64["u"])) - g["sum_u"]) < 1e-9


# ----------------------------------------------------------------------------- initial state

@pytest.mark.parametrize("zoh", [False, True])
def test_P6_initial_state_unrolled(zoh):
    # with h_0 given: y_t gains sum_n C_t[n] exp(A_n sum_{r<=t} Delta_r) h_0[n], and the end state
    # gains exp(A_n sum Delta) h_0[n]; the input terms are the unrolled double sum of P6
    rng = np.random.default_rng(13)
    batch, L, D, N, K = 2, 19, 3, 4, 2
    c = rand_case(rng, batch, L, D, N, K=K)
    h0 = rng.standard_normal((K, batch, D, N))
    out, last = oracle.selective_scan(c["u"], c["delta"], c["A"], c["B"], c["C"], Dskip=c["Dskip"],
                                      z=None, delta_bias=c["delta_bias"], softplus=True,
                                      dirs=(FWD, REV), zoh_exact=zoh, initial_state=h0)
    ref = np.zeros((batch, L, D))
    href = np.zeros((K, batch, D, N))
    for k in range(K):
        order = np.arange(L) if k == 0 else np.arange(L)[::-1]
        for b in range(batch):
            for d in range(D):
                dl = np_softplus(c["delta"][k, b, :, d] + c["delta_bias"][d])
                cum = np.concatenate([[0.0], np.cumsum(dl)])
                a = c["A"][d]
                for t in range(L):
                    decay0 = np.exp(a * cum[t + 1])
                    acc = np.sum(c["C"][k, b, t] * decay0 * h0[k, b, d])
                    for s in range(t + 1):
                        bbar = (np.expm1(dl[s] * a) / a) if zoh else dl[s]
                        acc += np.sum(c["C"][k, b, t] * np.exp(a * (cum[t + 1] - cum[s + 1])) *
                                      bbar * c["B"][k, b, s]) * c["u"][b, order[s], d]
                    ref[b, order[t], d] += acc + c["Dskip"][d] * c["u"][b, order[t], d]
                hh = np.exp(a * cum[L]) * h0[k, b, d]
                for s in range(L):
                    bbar = (np.expm1(dl[s] * a) / a) if zoh else dl[s]
                    hh = hh + np.exp(a * (cum[L] - cum[s + 1])) * bbar * c["B"][k, b, s] \
                        * c["u"][b, order[s], d]
                href[k, b, d] = hh
    assert rel_err(out, ref) < 1e-11
    assert rel_err(last, href) < 1e-11


def test_P7_initial_state_continues_a_split_scan():
    rng = np.random.default_rng(14)
    batch, L, D, N, T = 2, 30, 3, 5, 11
    c = rand_case(rng, batch, L, D, N)
    args = dict(Dskip=c["Dskip"], delta_bias=c["delta_bias"], softplus=True)
    out, last = oracle.selective_scan(c["u"], c["delta"], c["A"], c["B"], c["C"], z=c["z"], **args)
    _, h1 = oracle.selective_scan(c["u"][:, :T], c["delta"][:, :, :T], c["A"], c["B"][:, :, :T],
                                  c["C"][:, :, :T], z=c["z"][:, :T], **args)
    out2, last2 = oracle.selective_scan(c["u"][:, T:], c["delta"][:, :, T:], c["A"],
                                        c["B"][:, :, T:], c["C"][:, :, T:], z=c["z"][:, T:],
                                        initial_state=h1, **args)
    assert rel_err(out2, out[:, T:]) < 1e-13
    assert rel_err(last2, last) < 1e-13
    e = np.zeros((batch, 0, D))
    _, l0 = oracle.selective_scan(e, np.zeros((1, batch, 0, D)), c["A"], np.zeros((1, batch, 0, N)),
                                  np.zeros((1, batch, 0, N)), initial_state=h1)
    assert np.array_equal(l0, h1)


# ----------------------------------------------------------------------------- P9, P10 (conv)

def _np_conv_silu(u, w, cb, kind, H, W):
    """[batch, L, D] in the scan order of `kind`: numpy's convolution of the permuted sequence
    with the taps reversed (np.convolve flips its kernel), cut to the first L outputs, plus the
    bias, then x * sigmoid(x)."""
    order = _perm_by_loops(kind, H, W)
    seq = u[:, order]
    L = seq.shape[1]
    out = np.empty_like(seq)
    for b in range(seq.shape[0]):
        for d in range(seq.shape[2]):
            c = np.convolve(seq[b, :, d], w[d, ::-1])[:L] + cb[d]
            out[b, :, d] = c / (1.0 + np.exp(-c))
    return out, order


CONV_CASES = [((FWD,), 1, 23, 4), ((FWD, REV), 1, 29, 4), ((FWD, COL, REV, COLREV), 5, 7, 4),
              ((COLREV, FWD), 3, 4, 2), ((REV,), 1, 9, 1), ((COL,), 4, 3, 3)]


@pytest.mark.parametrize("dirs,H,W,width", CONV_CASES)
def test_P9_conv_equals_numpy_convolution(dirs, H, W, width):
    rng = np.random.default_rng(40 + width + len(dirs))
    batch, L, D, K = 2, H * W, 3, len(dirs)
    u = rng.standard_normal((batch, L, D))
    w = rng.standard_normal((K, D, width))
    cb = rng.standard_normal((K, D))
    got = oracle.conv_silu(u, w, cb, dirs=dirs, H=H, W=W)
    for k, kind in enumerate(dirs):
        ref, _ = _np_conv_silu(u, w[k], cb[k], kind, H, W)
        assert rel_err(got[k], ref) < 1e-13
    # no bias given reads as zero
    got0 = oracle.conv_silu(u, w, None, dirs=dirs, H=H, W=W)
    ref0, _ = _np_conv_silu(u, w[0], np.zeros(D), dirs[0], H, W)
    assert rel_err(got0[0], ref0) < 1e-13


@pytest.mark.parametrize("dirs,H,W,width", CONV_CASES)
def test_P10_conv_scan_equals_scans_of_convolved_inputs(dirs, H, W, width):
    rng = np.random.default_rng(60 + width + len(dirs))
    batch, L, D, N, K = 2, H * W, 3, 4, len(dirs)
    c = rand_case(rng, batch, L, D, N, K=K)
    w = rng.standard_normal((K, D, width))
    cb = rng.standard_normal((K, D))
    args = dict(Dskip=c["Dskip"], delta_bias=c["delta_bias"], softplus=True)
    out, last = oracle.selective_scan(c["u"], c["delta"], c["A"], c["B"], c["C"], z=c["z"],
                                      dirs=dirs, H=H, W=W, conv_weight=w, conv_bias=cb, **args)
    total = np.zeros_like(c["u"])
    lasts = []
    for k, kind in enumerate(dirs):
        u_scan, order = _np_conv_silu(c["u"], w[k], cb[k], kind, H, W)
        u_sp = np.empty_like(u_scan)
        u_sp[:, order] = u_scan                         # the convolved input at its position
        y_k, l_k = oracle.selective_scan(u_sp, c["delta"][k:k + 1], c["A"], c["B"][k:k + 1],
                                         c["C"][k:k + 1], z=None, dirs=(kind,), H=H, W=W, **args)
        total += y_k
        lasts.append(l_k[0])
    gate = c["z"] / (1.0 + np.exp(-c["z"]))
    assert rel_err(out, total * gate) < 1e-12
    assert rel_err(last, np.stack(lasts)) < 1e-12


# ----------------------------------------------------------------------------- P11 (input per direction)

@pytest.mark.parametrize("dirs,H,W,width", [((FWD, COL, REV, COLREV), 5, 7, 0),
                                            ((FWD, REV), 1, 19, 4), ((FWD, FWD), 1, 23, 0),
                                            ((COL, FWD, REV), 4, 6, 3)])
def test_P11_input_per_direction_is_a_sum_of_scans(dirs, H, W, width):
    rng = np.random.default_rng(80 + len(dirs) + width)
    batch, L, D, N, K = 2, H * W, 3, 4, len(dirs)
    c = rand_case(rng, batch, L, D, N, K=K)
    u = rng.standard_normal((K, batch, L, D))
    conv = {}
    if width:
        conv = dict(conv_weight=rng.standard_normal((K, D, width)),
                    conv_bias=rng.standard_normal((K, D)))
    args = dict(Dskip=c["Dskip"], delta_bias=c["delta_bias"], softplus=True, H=H, W=W)
    out, last = oracle.selective_scan(u, c["delta"], c["A"], c["B"], c["C"], z=c["z"], dirs=dirs,
                                      **conv, **args)
    total = np.zeros((batch, L, D))
    lasts = []
    for k, kind in enumerate(dirs):
        conv_k = {key: v[k:k + 1] for key, v in conv.items()}
        y_k, l_k = oracle.selective_scan(u[k], c["delta"][k:k + 1], c["A"], c["B"][k:k + 1],
                                         c["C"][k:k + 1], z=None, dirs=(kind,), **conv_k, **args)
        total += y_k
        lasts.append(l_k[0])
    gate = c["z"] / (1.0 + np.exp(-c["z"]))
    assert rel_err(out, total * gate) < 1e-13
    assert np.array_equal(last, np.stack(lasts))


def test_P11_cromb_cross_modal_scan():
    rng = np.random.default_rng(90)
    batch, L, D, N = 2, 31, 4, 5
    x_rgb, x_depth = rng.standard_normal((2, batch, L, D))
    d_rgb, d_depth = rng.standard_normal((2, 1, batch, L, D))
    B_rgb, B_depth, C_rgb, C_depth = rng.standard_normal((4, 1, batch, L, N))
    A = -rng.uniform(0.1, 2.0, size=(D, N))
    Dskip = rng.standard_normal(D)
    bias = rng.uniform(-2.0, 0.5, size=D)
    args = dict(Dskip=Dskip, delta_bias=bias, softplus=True, z=None)
    out_rgb, _ = oracle.selective_scan(x_rgb, d_rgb, A, B_rgb, C_depth, **args)
    out_depth, _ = oracle.selective_scan(x_depth, d_depth, A, B_depth, C_rgb, **args)
    out, _ = oracle.selective_scan(np.stack([x_rgb, x_depth]), np.concatenate([d_rgb, d_depth]), A,
                                   np.concatenate([B_rgb, B_depth]),
                                   np.concatenate([C_depth, C_rgb]), dirs=(FWD, FWD), **args)
    assert rel_err(out, out_rgb + out_depth) < 1e-13


# ----------------------------------------------------------------------------- P12 (int8 Delta)

@pytest.mark.parametrize("softplus", [True, False])
def test_P12_int8_delta_codes_with_channel_scales(softplus):
    rng = np.random.default_rng(95)
    batch, L, D, N, K = 2, 27, 5, 4, 2
    c = rand_case(rng, batch, L, D, N, K=K)
    q = rng.integers(-127, 128, size=(K, batch, L, D)).astype(np.float64)
    scale = rng.uniform(0.002, 0.05, size=D).astype(np.float32).astype(np.float64)
    args = dict(Dskip=c["Dskip"], delta_bias=c["delta_bias"], softplus=softplus, z=c["z"],
                dirs=(FWD, REV))
    out, last = oracle.selective_scan(c["u"], q, c["A"], c["B"], c["C"], delta_scale=scale, **args)
    raw = q * scale[None, None, None, :]              # exact: 8-bit codes times 24-bit scales
    ref, ref_last = oracle.selective_scan(c["u"], raw, c["A"], c["B"], c["C"], **args)
    assert np.array_equal(out, ref) and np.array_equal(last, ref_last)
    # and a scale is not an offset: scaling the codes by 2 and halving the scale is the same scan
    out2, _ = oracle.selective_scan(c["u"], 2 * q, c["A"], c["B"], c["C"], delta_scale=scale / 2,
                                    **args)
    assert np.array_equal(out2, out)


# ----------------------------------------------------------------------------- P13 (parameters per direction)

@pytest.mark.parametrize("dirs,H,W", [((FWD, REV), 1, 21), ((FWD, COL, REV, COLREV), 4, 5)])
def test_P13_parameters_per_direction(dirs, H, W):
    rng = np.random.default_rng(99 + len(dirs))
    batch, L, D, N, K = 2, H * W, 3, 4, len(dirs)
    c = rand_case(rng, batch, L, D, N, K=K)
    A = -rng.uniform(0.1, 2.0, size=(K, D, N))
    Dskip = rng.standard_normal((K, D))
    bias = rng.uniform(-2.0, 0.5, size=(K, D))
    out, last = oracle.selective_scan(c["u"], c["delta"], A, c["B"], c["C"], Dskip=Dskip,
                                      z=c["z"], delta_bias=bias, dirs=dirs, H=H, W=W)
    total = np.zeros_like(c["u"])
    lasts = []
    for k, kind in enumerate(dirs):
        y_k, l_k = oracle.selective_scan(c["u"], c["delta"][k:k + 1], A[k], c["B"][k:k + 1],
                                         c["C"][k:k + 1], Dskip=Dskip[k], z=None,
                                         delta_bias=bias[k], dirs=(kind,), H=H, W=W)
        total += y_k
        lasts.append(l_k[0])
    gate = c["z"] / (1.0 + np.exp(-c["z"]))
    assert rel_err(out, total * gate) < 1e-13
    assert np.array_equal(last, np.stack(lasts))
