"""Pins for the CPU oracle: checks against things other than the oracle itself.

Every pin takes an ``oracle.Oracle`` (the default build, or a build with one
planted mistake) and raises ``AssertionError`` when the oracle disagrees with:

* a hand-worked example (``tests/golden/*.txt``, each with its derivation),
* a closed form (decay-only run, dt -> 0, C = 0),
* the quadratic "SSD dual" form of the recurrence on tiny shapes, evaluated
  independently with numpy (no loop over the recurrence),
* a library routine (numpy float32 rounding, ``numpy.logaddexp`` for softplus,
  ``scipy.special.expit`` for the sigmoid, ``numpy`` mat-vec products),
* brute force (exact nearest-bfloat16 search with rationals),
* invariants: linearity in (S0, x), group partition, slot-independence of the
  per-sequence computation, T=1 scan equals one step, T-token scan equals T
  steps.

The pins are chosen so that a plausible mistake anywhere in the oracle (a
dropped term, a wrong sign or index, a transposed operand, a wrong rounding)
fails at least one of them; ``test_oracle_mutants.py`` checks exactly that.
"""

from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np
from scipy.special import expit

import oracle as O

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read_golden(name: str) -> dict:
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            k, v = (s.strip() for s in line.split("=", 1))
            vals = [float(t) for t in v.split()]
            out[k] = vals[0] if len(vals) == 1 else np.array(vals)
    return out


def _rng(seed: int) -> np.random.Generator:
    return np.random.default_rng(seed)


# ------------------------------------------------------------------ rounding

def _bf16_candidates(x: float):
    """bfloat16 values around x (bit patterns near the float32 truncation)."""
    u = int(np.array([x], dtype=np.float32).view(np.uint32)[0]) & 0xFFFF0000
    cands = []
    for d in (-2, -1, 0, 1, 2):
        b = (u + d * 0x10000) & 0xFFFFFFFF
        v = float(np.array([b], dtype=np.uint32).view(np.float32)[0])
        if math.isfinite(v):
            cands.append((v, (b >> 16) & 1))
    return cands


def _nearest_bf16_brute(x: float) -> float:
    fx = Fraction(x)
    best = None
    for v, odd in _bf16_candidates(x):
        d = abs(Fraction(v) - fx)
        key = (d, odd)  # ties go to the even significand
        if best is None or key < best[0]:
            best = (key, v)
    return best[1]


def pin_round_bf16_brute(orc: O.Oracle) -> None:
    """bfloat16 rounding = exact nearest bfloat16, ties to even (brute force)."""
    rng = _rng(1)
    xs = list(rng.normal(size=300) * 10.0 ** rng.integers(-8, 8, size=300))
    # exact midpoints between neighbouring bfloat16 values, both parities
    for base in (1.0, 1.0078125, -3.140625, 0.0001220703125):
        ulp = 2.0 ** (math.frexp(abs(base))[1] - 1 - 7)
        xs += [base + ulp / 2, base - ulp / 2, base + 1.5 * ulp]
    for x in xs:
        got = orc.round_bf16(float(x))
        want = _nearest_bf16_brute(float(x))
        assert got == want, (x, got, want)


def _nearest_f16_brute(x: float) -> float:
    """Exact nearest binary16 (ties to even) by searching the neighbours of
    numpy's conversion over rationals."""
    h = np.array([x], dtype=np.float64).astype(np.float16)
    u = int(h.view(np.uint16)[0])
    fx = Fraction(x)
    best = None
    for d in (-2, -1, 0, 1, 2):
        b = (u + d) & 0xFFFF
        v = float(np.array([b], dtype=np.uint16).view(np.float16)[0])
        if not math.isfinite(v):
            continue
        key = (abs(Fraction(v) - fx), b & 1)
        if best is None or key < best[0]:
            best = (key, v)
    return best[1]


def pin_round_f16_brute(orc: O.Oracle) -> None:
    """fp16 rounding = exact nearest binary16, ties to even, subnormals
    included (brute force), and numpy's float64 -> float16 in range."""
    rng = _rng(13)
    xs = list(rng.normal(size=300) * 10.0 ** rng.integers(-7, 5, size=300))
    for base in (1.0, 1.0009765625, -3.140625, 6.103515625e-05, 2.0 ** -20):
        ulp = 2.0 ** max(math.frexp(abs(base))[1] - 1 - 10, -24)
        xs += [base + ulp / 2, base - ulp / 2, base + 1.5 * ulp]
    for x in xs:
        got = orc.round_f16(float(x))
        assert got == _nearest_f16_brute(float(x)), x
        assert got == float(np.float16(x)), x
    assert math.isinf(orc.round_f16(70000.0)) and orc.round_f16(65504.0) == 65504.0


def pin_round_f32_library(orc: O.Oracle) -> None:
    """float32 rounding agrees with numpy's float64 -> float32 conversion."""
    rng = _rng(2)
    xs = rng.normal(size=500) * 10.0 ** rng.integers(-20, 20, size=500)
    for x in xs:
        assert orc.round_f32(float(x)) == float(np.float32(x))


# --------------------------------------------------------------- activations

def pin_softplus(orc: O.Oracle) -> None:
    """softplus against numpy.logaddexp(0, v), its inverse, and its limits.

    Above 20 the oracle returns v itself (the usual threshold); there the exact
    value differs by log1p(exp(-v)) < 2.1e-9, i.e. below 1.1e-10 relative.
    """
    for v in np.linspace(-30, 30, 241):
        want = float(np.logaddexp(0.0, v))
        if v <= 20.0:
            assert math.isclose(orc.softplus(v), want, rel_tol=1e-14, abs_tol=1e-300), v
        else:
            assert orc.softplus(v) == v and math.isclose(v, want, rel_tol=1.1e-10), v
    for u in np.linspace(1e-3, 0.1, 17):  # the inverse used for dt_bias
        assert math.isclose(orc.softplus(math.log(math.expm1(u))), u, rel_tol=1e-13)
    assert orc.softplus(-1e4) == 0.0
    assert orc.softplus(50.0) == 50.0


def pin_silu(orc: O.Oracle) -> None:
    for v in np.linspace(-20, 20, 161):
        assert math.isclose(orc.silu(v), v * float(expit(v)), rel_tol=1e-14, abs_tol=1e-300)


# ---------------------------------------------------------------------- conv

def pin_conv_hand(orc: O.Oracle) -> None:
    """Hand-worked K=4 conv over three tokens, two channels (golden file)."""
    g = read_golden("conv_k4_two_channels.txt")
    K = int(g["K"])
    w = np.stack([g["w0"], g["w1"]])
    cache = np.ascontiguousarray(np.stack([g["cache0"], g["cache1"]]).T)
    x = np.stack([g["x0"], g["x1"]]).T
    out = orc.conv1d(cache, x, w, g["bias"], activation=0)
    assert K == w.shape[1]
    assert np.array_equal(out[:, 0], g["out0"]) and np.array_equal(out[:, 1], g["out1"]), out
    assert np.array_equal(cache[:, 0], g["cache_after0"])
    assert np.array_equal(cache[:, 1], g["cache_after1"])


def pin_conv_one_hot_taps(orc: O.Oracle) -> None:
    """A one-hot weight at tap k delays the input by K-1-k tokens, exactly.

    Tap K-1 is the identity; tap 0 returns the input from K-1 tokens back,
    read from the cache for the first tokens. After T >= K-1 tokens the cache
    holds the last K-1 raw inputs bit for bit.
    """
    rng = _rng(3)
    K, C, T = 4, 5, 7
    x = rng.normal(size=(T, C))
    cache0 = rng.normal(size=(K - 1, C))
    hist = np.concatenate([cache0, x])  # row j = token j-(K-1)
    for k in range(K):
        w = np.zeros((C, K))
        w[:, k] = 1.0
        cache = cache0.copy()
        out = orc.conv1d(cache, x, w, None, activation=0)
        delay = K - 1 - k
        want = hist[K - 1 - delay: K - 1 - delay + T]
        assert np.array_equal(out, want), k
        assert np.array_equal(cache, x[T - (K - 1):])
    # short sequences: T < K-1 keeps part of the old cache
    cache = cache0.copy()
    orc.conv1d(cache, x[:1], np.zeros((C, K)), None, activation=0)
    assert np.array_equal(cache, np.concatenate([cache0[1:], x[:1]]))


def pin_conv_silu(orc: O.Oracle) -> None:
    """With activation the output is silu of the linear conv (scipy's expit)."""
    rng = _rng(4)
    K, C, T = 4, 6, 3
    x = rng.normal(size=(T, C))
    w = rng.normal(size=(C, K))
    b = rng.normal(size=C)
    c0 = rng.normal(size=(K - 1, C))
    lin = orc.conv1d(c0.copy(), x, w, b, activation=0)
    act = orc.conv1d(c0.copy(), x, w, b, activation=1)
    assert np.allclose(act, lin * expit(lin), rtol=1e-14, atol=0)


# ----------------------------------------------------------------- SSM step

def _random_problem(rng, H, P, N, G, T, s0_scale=1.0):
    cd = H * P + 2 * G * N
    return dict(
        S0=rng.normal(size=(H, P, N)) * s0_scale,
        xbc=rng.normal(size=(T, cd)),
        dt_raw=rng.normal(size=(T, H)),
        dt_bias=np.log(np.expm1(rng.uniform(1e-3, 0.1, size=H))),
        A_log=np.log(rng.uniform(1, 16, size=H)),
        D=rng.normal(size=H),
        z=rng.normal(size=(T, H * P)),
    )


def _scan(orc, pr, G, round_mode=O.ROUND_NONE, with_z=True, S0=None):
    S = np.array(pr["S0"] if S0 is None else S0, dtype=np.float64, copy=True)
    y = orc.ssm_scan(S, round_mode, pr["xbc"], pr["dt_raw"], pr["dt_bias"], pr["A_log"], pr["D"],
                     pr["z"] if with_z else None, G)
    return S, y


def pin_ssm_hand(orc: O.Oracle) -> None:
    """Hand-worked single step (golden file), with and without the gate."""
    g = read_golden("ssm_step_hand.txt")
    ln2 = math.log(2.0)
    H, P, N, G = 1, 2, 2, 1
    xbc = np.concatenate([g["x"], g["B"], g["C"]])
    args = (xbc, [g["dt_raw"]], [g["dt_bias"]], [g["A_log"]], [g["D"]])
    S = np.array(g["S"], dtype=np.float64).reshape(H, P, N)
    y = orc.ssm_step(S, O.ROUND_NONE, *args, None, G)
    want_S = g["S_new_a"] + g["S_new_b"] * ln2
    want_y = g["y_a"] + g["y_b"] * ln2
    assert np.allclose(S.ravel(), want_S, rtol=1e-14, atol=1e-15), (S.ravel(), want_S)
    assert np.allclose(y, want_y, rtol=1e-14, atol=1e-15), (y, want_y)
    S = np.array(g["S"], dtype=np.float64).reshape(H, P, N)
    y = orc.ssm_step(S, O.ROUND_NONE, *args, np.zeros(P), G)
    assert np.array_equal(y, np.zeros(P))


def pin_decay_only_closed_form(orc: O.Oracle) -> None:
    """B = 0: after T steps S_T = S_0 * exp(-exp(A_log) * sum_t dt_t).

    With dt_raw = 0 the step size is softplus(dt_bias) = u, where dt_bias was
    drawn as log(expm1(u)); the closed form uses u * T directly.
    """
    rng = _rng(5)
    H, P, N, G, T = 4, 3, 5, 2, 6
    pr = _random_problem(rng, H, P, N, G, T)
    u = rng.uniform(1e-3, 0.1, size=H)
    pr["dt_bias"] = np.log(np.expm1(u))
    pr["dt_raw"][:] = 0.0
    pr["xbc"][:, H * P:H * P + G * N] = 0.0  # B = 0
    S, _ = _scan(orc, pr, G)
    want = pr["S0"] * np.exp(-np.exp(pr["A_log"]) * u * T)[:, None, None]
    assert np.allclose(S, want, rtol=1e-12, atol=0), np.max(np.abs(S - want))
    # one step, storage rounding: S' = round(S * dA) exactly
    S1 = pr["S0"].copy()
    orc.ssm_step(S1, O.ROUND_NONE, pr["xbc"][0], pr["dt_raw"][0], pr["dt_bias"], pr["A_log"],
                 pr["D"], None, G)
    dA = np.exp(-np.exp(pr["A_log"]) * u)
    assert np.allclose(S1, pr["S0"] * dA[:, None, None], rtol=1e-13, atol=0)


def pin_dt_to_zero_identity(orc: O.Oracle) -> None:
    """dt_raw = -1e4 gives dt = 0 exactly: S' == S bitwise, y = C.S + D.x."""
    rng = _rng(6)
    H, P, N, G = 4, 3, 5, 2
    pr = _random_problem(rng, H, P, N, G, 1)
    pr["dt_raw"][:] = -1e4
    for round_mode in (O.ROUND_NONE, O.ROUND_F32, O.ROUND_BF16):
        S0 = orc.round_array(pr["S0"], round_mode).reshape(H, P, N)
        S = S0.copy()
        y = orc.ssm_step(S, round_mode, pr["xbc"][0], pr["dt_raw"][0], pr["dt_bias"], pr["A_log"],
                         pr["D"], None, G)
        assert np.array_equal(S, S0)
        x = pr["xbc"][0, :H * P].reshape(H, P)
        Cm = pr["xbc"][0, H * P + G * N:].reshape(G, N)
        hpg = H // G
        want = np.stack([S0[h] @ Cm[h // hpg] + pr["D"][h] * x[h] for h in range(H)]).ravel()
        assert np.allclose(y, want, rtol=1e-13, atol=1e-14)
        yz = orc.ssm_step(S0.copy(), round_mode, pr["xbc"][0], pr["dt_raw"][0], pr["dt_bias"],
                          pr["A_log"], pr["D"], pr["z"][0], G)
        assert np.allclose(yz, want * pr["z"][0] * expit(pr["z"][0]), rtol=1e-13, atol=1e-14)


def pin_c_zero(orc: O.Oracle) -> None:
    """C = 0: y = D * x exactly (no gate), whatever the state does."""
    rng = _rng(7)
    H, P, N, G = 4, 3, 5, 2
    pr = _random_problem(rng, H, P, N, G, 1)
    pr["xbc"][0, H * P + G * N:] = 0.0
    S = pr["S0"].copy()
    y = orc.ssm_step(S, O.ROUND_NONE, pr["xbc"][0], pr["dt_raw"][0], pr["dt_bias"], pr["A_log"],
                     pr["D"], None, G)
    x = pr["xbc"][0, :H * P].reshape(H, P)
    assert np.array_equal(y, (pr["D"][:, None] * x).ravel())


def _dual_form(pr, H, P, N, G):
    """Quadratic (SSD dual) form: y and S_T from closed sums, no recurrence loop.

    y_t = sum_{u<=t} (C_t . B_u) exp(A (c_t - c_u)) dt_u x_u
          + exp(A c_t) (S_0 C_t) + D x_t,
    S_T = sum_u exp(A (c_T - c_u)) dt_u x_u B_u^T + exp(A c_T) S_0,
    with c_t = dt_1 + ... + dt_t, per head, and B, C of the head's group.
    """
    T = pr["xbc"].shape[0]
    hp = H * P
    hpg = H // G
    x = pr["xbc"][:, :hp].reshape(T, H, P)
    Bm = pr["xbc"][:, hp:hp + G * N].reshape(T, G, N)
    Cm = pr["xbc"][:, hp + G * N:].reshape(T, G, N)
    y = np.zeros((T, H, P))
    S = np.zeros((H, P, N))
    for h in range(H):
        g = h // hpg
        dt = np.logaddexp(0.0, pr["dt_raw"][:, h] + pr["dt_bias"][h])
        a = -np.exp(pr["A_log"][h])
        c = np.cumsum(dt)
        L = np.exp(a * (c[:, None] - c[None, :])) * np.tril(np.ones((T, T)))
        CB = Cm[:, g, :] @ Bm[:, g, :].T                 # [t, u]
        M = CB * L * dt[None, :]
        y[:, h, :] = M @ x[:, h, :] + np.exp(a * c)[:, None] * (Cm[:, g, :] @ pr["S0"][h].T) \
            + pr["D"][h] * x[:, h, :]
        w = np.exp(a * (c[-1] - c)) * dt                 # [u]
        S[h] = (x[:, h, :] * w[:, None]).T @ Bm[:, g, :] + np.exp(a * c[-1]) * pr["S0"][h]
    return y.reshape(T, hp), S


def pin_quadratic_dual_form(orc: O.Oracle) -> None:
    """The scan equals the quadratic SSD form on tiny shapes, to 1e-12."""
    rng = _rng(8)
    for (H, P, N, G, T) in [(1, 1, 1, 1, 1), (2, 3, 4, 1, 5), (4, 2, 3, 2, 8), (4, 4, 4, 2, 7),
                            (3, 2, 4, 3, 4)]:
        pr = _random_problem(rng, H, P, N, G, T)
        S, y = _scan(orc, pr, G, with_z=False)
        y_ref, S_ref = _dual_form(pr, H, P, N, G)
        scale_y = max(1.0, np.max(np.abs(y_ref)))
        scale_S = max(1.0, np.max(np.abs(S_ref)))
        assert np.max(np.abs(y - y_ref)) <= 1e-12 * scale_y, (H, P, N, G, T)
        assert np.max(np.abs(S - S_ref)) <= 1e-12 * scale_S, (H, P, N, G, T)


def pin_linearity(orc: O.Oracle) -> None:
    """With dt, B, C fixed: S_T(S0, x) = S_T(S0, 0) + S_T(0, x); scaling by alpha."""
    rng = _rng(9)
    H, P, N, G, T = 4, 3, 5, 2, 6
    pr = _random_problem(rng, H, P, N, G, T)
    hp = H * P
    S_full, y_full = _scan(orc, pr, G, with_z=False)
    pr0 = dict(pr, xbc=pr["xbc"].copy())
    pr0["xbc"][:, :hp] = 0.0
    S_a, y_a = _scan(orc, pr0, G, with_z=False)
    S_b, y_b = _scan(orc, pr, G, with_z=False, S0=np.zeros_like(pr["S0"]))
    assert np.allclose(S_full, S_a + S_b, rtol=1e-12, atol=1e-13)
    assert np.allclose(y_full, y_a + y_b, rtol=1e-12, atol=1e-13)
    alpha = 2.5
    pr2 = dict(pr, xbc=pr["xbc"].copy())
    pr2["xbc"][:, :hp] *= alpha
    S_s, y_s = _scan(orc, pr2, G, with_z=False, S0=alpha * pr["S0"])
    assert np.allclose(S_s, alpha * S_full, rtol=1e-12, atol=1e-13)
    assert np.allclose(y_s, alpha * y_full, rtol=1e-12, atol=1e-13)


def pin_group_partition(orc: O.Oracle) -> None:
    """A G-group run equals G independent one-group runs on the head slices."""
    rng = _rng(10)
    H, P, N, G, T = 8, 2, 3, 4, 3
    hpg = H // G
    pr = _random_problem(rng, H, P, N, G, T)
    S, y = _scan(orc, pr, G)
    hp = H * P
    Bm = pr["xbc"][:, hp:hp + G * N].reshape(T, G, N)
    Cm = pr["xbc"][:, hp + G * N:].reshape(T, G, N)
    x = pr["xbc"][:, :hp].reshape(T, H, P)
    z = pr["z"].reshape(T, H, P)
    for g in range(G):
        hs = slice(g * hpg, (g + 1) * hpg)
        sub = dict(
            S0=pr["S0"][hs].copy(),
            xbc=np.concatenate([x[:, hs].reshape(T, -1), Bm[:, g], Cm[:, g]], axis=1),
            dt_raw=pr["dt_raw"][:, hs], dt_bias=pr["dt_bias"][hs], A_log=pr["A_log"][hs],
            D=pr["D"][hs], z=z[:, hs].reshape(T, -1))
        S_g, y_g = _scan(orc, sub, 1)
        assert np.array_equal(S_g, S[hs])
        assert np.array_equal(y_g, y.reshape(T, H, P)[:, hs].reshape(T, -1))


def pin_scan_is_steps(orc: O.Oracle) -> None:
    """A T=1 scan equals one step (any rounding); a T-token scan equals T steps."""
    rng = _rng(11)
    H, P, N, G, T = 4, 3, 5, 2, 5
    pr = _random_problem(rng, H, P, N, G, T)
    for rm in (O.ROUND_NONE, O.ROUND_F32, O.ROUND_BF16):
        S0 = orc.round_array(pr["S0"], rm).reshape(H, P, N)
        pr1 = dict(pr, xbc=pr["xbc"][:1], dt_raw=pr["dt_raw"][:1], z=pr["z"][:1])
        S_scan, y_scan = _scan(orc, pr1, G, round_mode=rm, S0=S0)
        S_step = S0.copy()
        y_step = orc.ssm_step(S_step, rm, pr["xbc"][0], pr["dt_raw"][0], pr["dt_bias"],
                              pr["A_log"], pr["D"], pr["z"][0], G)
        assert np.array_equal(S_scan, S_step) and np.array_equal(y_scan[0], y_step)
    S_scan, y_scan = _scan(orc, pr, G)
    S = pr["S0"].copy()
    for t in range(T):
        y_t = orc.ssm_step(S, O.ROUND_NONE, pr["xbc"][t], pr["dt_raw"][t], pr["dt_bias"],
                           pr["A_log"], pr["D"], pr["z"][t], G)
        assert np.array_equal(y_t, y_scan[t])
    assert np.array_equal(S, S_scan)


def pin_state_rounding_on_store(orc: O.Oracle) -> None:
    """A stored step rounds the new state once to the storage precision, and y
    comes from the unrounded state: compare with a ROUND_NONE step."""
    rng = _rng(12)
    H, P, N, G = 2, 3, 4, 1
    pr = _random_problem(rng, H, P, N, G, 1)
    for rm in (O.ROUND_F32, O.ROUND_BF16):
        S0 = orc.round_array(pr["S0"], rm).reshape(H, P, N)
        S_exact = S0.copy()
        y_exact = orc.ssm_step(S_exact, O.ROUND_NONE, pr["xbc"][0], pr["dt_raw"][0],
                               pr["dt_bias"], pr["A_log"], pr["D"], None, G)
        S_r = S0.copy()
        y_r = orc.ssm_step(S_r, rm, pr["xbc"][0], pr["dt_raw"][0], pr["dt_bias"], pr["A_log"],
                           pr["D"], None, G)
        assert np.array_equal(y_r, y_exact)
        if rm == O.ROUND_F32:
            assert np.array_equal(S_r, S_exact.astype(np.float32).astype(np.float64))
        else:
            assert np.array_equal(S_r.ravel(), [_nearest_bf16_brute(v) for v in S_exact.ravel()])


# ------------------------------------------------------------ gated RMSNorm

def pin_rmsnorm_hand(orc: O.Oracle) -> None:
    """Hand-worked example, tests/golden/group_rmsnorm_hand.txt (two groups,
    eps = 0 and eps = 1, non-unit weights)."""
    g = read_golden("group_rmsnorm_hand.txt")
    for eps, tag in ((0.0, "eps0"), (1.0, "eps1")):
        out = orc.group_rmsnorm(g["v"], int(g["G"]), eps, g["w"])
        want = g[f"{tag}_coef"] * np.sqrt(g[f"{tag}_root"])
        assert np.allclose(out, want, rtol=1e-14, atol=0), (tag, out, want)


def pin_rmsnorm_unit_rms(orc: O.Oracle) -> None:
    """With unit weights and eps = 0 every group of the output has root mean
    square exactly 1 and is a positive multiple of the input group."""
    rng = _rng(71)
    G, L = 4, 16
    v = rng.normal(size=G * L) * rng.uniform(0.1, 10.0, size=G).repeat(L)
    out = orc.group_rmsnorm(v, G, 0.0, np.ones(G * L))
    for gi in range(G):
        o, x = out[gi * L:(gi + 1) * L], v[gi * L:(gi + 1) * L]
        assert abs(np.mean(o * o) - 1.0) < 1e-12
        ratio = o / x
        assert np.all(ratio > 0) and np.ptp(ratio) < 1e-12 * np.max(ratio)


def pin_rmsnorm_scale_sign(orc: O.Oracle) -> None:
    """eps = 0: the output does not change when a row is scaled by a positive
    factor, and changes sign with the row."""
    rng = _rng(72)
    G, L = 2, 8
    v = rng.normal(size=G * L)
    w = rng.normal(size=G * L)
    base = orc.group_rmsnorm(v, G, 0.0, w)
    assert np.allclose(orc.group_rmsnorm(2.5 * v, G, 0.0, w), base, rtol=1e-13, atol=0)
    assert np.array_equal(orc.group_rmsnorm(-v, G, 0.0, w), -base)


def pin_rmsnorm_group_partition(orc: O.Oracle) -> None:
    """A G-group row is G independent one-group rows, bit for bit."""
    rng = _rng(73)
    G, L = 4, 8
    v = rng.normal(size=G * L)
    w = rng.normal(size=G * L)
    full = orc.group_rmsnorm(v, G, 1e-5, w)
    for gi in range(G):
        sl = slice(gi * L, (gi + 1) * L)
        assert np.array_equal(full[sl], orc.group_rmsnorm(v[sl], 1, 1e-5, w[sl]))


def pin_rmsnorm_eps_dominates(orc: O.Oracle) -> None:
    """When eps is far above the mean square, out = v * w / sqrt(eps)."""
    rng = _rng(74)
    G, L = 2, 8
    v = 1e-9 * rng.normal(size=G * L)
    w = rng.normal(size=G * L)
    out = orc.group_rmsnorm(v, G, 4.0, w)
    assert np.allclose(out, v * w / 2.0, rtol=1e-9, atol=0)


ALL_PINS = [
    pin_round_bf16_brute,
    pin_round_f16_brute,
    pin_round_f32_library,
    pin_softplus,
    pin_silu,
    pin_conv_hand,
    pin_conv_one_hot_taps,
    pin_conv_silu,
    pin_ssm_hand,
    pin_decay_only_closed_form,
    pin_dt_to_zero_identity,
    pin_c_zero,
    pin_quadratic_dual_form,
    pin_linearity,
    pin_group_partition,
    pin_scan_is_steps,
    pin_state_rounding_on_store,
    pin_rmsnorm_hand,
    pin_rmsnorm_unit_rms,
    pin_rmsnorm_scale_sign,
    pin_rmsnorm_group_partition,
    pin_rmsnorm_eps_dominates,
]
