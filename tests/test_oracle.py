"""Pins for the fp64 oracle, against facts other than the oracle itself.

Each check follows from the linear-attention definition on page
"MiniMax-M1で理解する：大規模言語モデルのコンテキスト長限界を突破する革新的アーキテクチャ"
(zenn.dev), section "線形アテンションの数学的基礎" (S_t = S_{t-1} + k_t v_t^T,
o_t = q_t S_t), from its factorised form phi(Q)(phi(K)^T V), or from plain
linear algebra: a hand-worked fixture, brute force over token pairs, closed
forms through numpy, integer exactness and invariants.  The mutant tests at
the end plant plausible mistakes in copies of the oracle's formulas and show
that these pins reject them.
"""
import os

import numpy as np
import pytest

import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _read_golden(name):
    rows = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            rows[key] = np.array([float(x) for x in vals])
    return rows


def _rel(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


# ---------------------------------------------------------------- fixtures
def test_hand_worked_example(oracle_mod):
    g = _read_golden("hand_worked_n3_d2.txt")
    q = g["q"].reshape(1, 3, 2)
    k = g["k"].reshape(1, 3, 2)
    v = g["v"].reshape(1, 3, 2)
    for fn in (oracle_mod.recurrent, oracle_mod.quadratic):
        o, s = fn(q, k, v)
        np.testing.assert_array_equal(o.reshape(-1), g["A.o"])
        np.testing.assert_array_equal(s.reshape(-1), g["A.S"])
        s0 = g["B.S0"].reshape(1, 2, 2)
        o, s = fn(q, k, v, s0)
        np.testing.assert_array_equal(o.reshape(-1), g["B.o"])
        np.testing.assert_array_equal(s.reshape(-1), g["B.S"])


def _brute(q, k, v, s0):
    """o_t = sum_{s<=t} (q_t . k_s) v_s + q_t S0 and S_N = S0 + sum_s k_s^T v_s,
    written as explicit pure-Python loops over token pairs."""
    N, dk = q.shape
    dv = v.shape[1]
    o = [[0.0] * dv for _ in range(N)]
    for t in range(N):
        for s in range(t + 1):
            a = sum(float(q[t, i]) * float(k[s, i]) for i in range(dk))
            for j in range(dv):
                o[t][j] += a * float(v[s, j])
        for j in range(dv):
            o[t][j] += sum(float(q[t, i]) * float(s0[i, j]) for i in range(dk))
    S = [[float(s0[i, j]) + sum(float(k[s, i]) * float(v[s, j]) for s in range(N))
          for j in range(dv)] for i in range(dk)]
    return np.array(o), np.array(S)


@pytest.mark.parametrize("N,dk,dv", [(1, 3, 2), (2, 4, 4), (5, 3, 6), (8, 8, 8), (7, 2, 5)])
@pytest.mark.parametrize("with_s0", [False, True])
def test_brute_force_small(oracle_mod, N, dk, dv, with_s0):
    q = _rand((N, dk), 1)
    k = _rand((N, dk), 2)
    v = _rand((N, dv), 3)
    s0 = _rand((dk, dv), 4) if with_s0 else np.zeros((dk, dv))
    ob, sb = _brute(q, k, v, s0)
    for fn in (oracle_mod.recurrent, oracle_mod.quadratic):
        o, s = fn(q[None], k[None], v[None], s0[None] if with_s0 else None)
        assert _rel(o[0], ob) < 1e-13
        assert _rel(s[0], sb) < 1e-13


@pytest.mark.parametrize("N,d", [(256, 64), (300, 128), (129, 128), (1024, 64)])
def test_recurrent_equals_quadratic(oracle_mod, N, d):
    q, k, v = synth.qkv((2, 2, N, d), d, "fp32", seed=N + d)
    s0 = _rand((2, 2, d, d), 7)
    o1, s1 = oracle_mod.recurrent(q, k, v, s0)
    o2, s2 = oracle_mod.quadratic(q, k, v, s0)
    assert _rel(o1, o2) < 1e-12
    assert _rel(s1, s2) < 1e-12


def test_first_output_invariant(oracle_mod):
    """o_1 = (q_1 . k_1) v_1 with a zero initial state; o_1 = q_1 S0 + (q_1 . k_1) v_1 otherwise."""
    q, k, v = synth.qkv((3, 5, 64), 64, "fp32", seed=11)
    o, _ = oracle_mod.recurrent(q, k, v)
    qn, kn, vn = (x.double().numpy() for x in (q, k, v))
    want = np.einsum("ui,ui->u", qn[:, 0], kn[:, 0])[:, None] * vn[:, 0]
    assert _rel(o[:, 0], want) < 1e-14
    s0 = _rand((3, 64, 64), 5)
    o, _ = oracle_mod.recurrent(q, k, v, s0)
    want2 = want + np.einsum("ui,uij->uj", qn[:, 0], s0)
    assert _rel(o[:, 0], want2) < 1e-14


def test_integer_inputs_exact(oracle_mod):
    """Inputs in {-1,0,1}: every partial sum is a small integer, so both forms are exact."""
    shape = (2, 3, 200, 16)
    q = synth.integer_valued(shape, seed=1)
    k = synth.integer_valued(shape, seed=2)
    v = synth.integer_valued(shape, seed=3)
    s0 = synth.integer_valued((2, 3, 16, 16), seed=4, lo=-3, hi=3)
    o1, s1 = oracle_mod.recurrent(q, k, v, s0)
    o2, s2 = oracle_mod.quadratic(q, k, v, s0)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(s1, s2)
    assert np.all(o1 == np.round(o1))
    # exact brute force on one unit
    ob, sb = _brute(q[1, 2].numpy(), k[1, 2].numpy(), v[1, 2].numpy(), s0[1, 2].numpy())
    np.testing.assert_array_equal(o1[1, 2], ob)
    np.testing.assert_array_equal(s1[1, 2], sb)


def test_final_state_is_library_gemm(oracle_mod):
    """S_N = S0 + K^T V, checked against numpy's matmul."""
    q, k, v = synth.qkv((4, 333, 32), 48, "fp32", seed=3)
    s0 = _rand((4, 32, 48), 9)
    _, s = oracle_mod.recurrent(q, k, v, s0)
    kn, vn = k.double().numpy(), v.double().numpy()
    want = s0 + np.matmul(kn.transpose(0, 2, 1), vn)
    assert _rel(s, want) < 1e-13


def test_ones_value_is_cumsum(oracle_mod):
    """With V = 1, every output column equals q_t . (k_1 + ... + k_t)."""
    N, d = 180, 24
    q = _rand((1, N, d), 1)
    k = _rand((1, N, d), 2)
    v = np.ones((1, N, 5))
    o, _ = oracle_mod.recurrent(q, k, v)
    want = np.einsum("ti,ti->t", q[0], np.cumsum(k[0], axis=0))
    for j in range(5):
        assert _rel(o[0, :, j], want) < 1e-13


def test_linearity_and_causality(oracle_mod):
    N, d = 97, 16
    q = _rand((1, N, d), 1)
    k = _rand((1, N, d), 2)
    v1 = _rand((1, N, d), 3)
    v2 = _rand((1, N, d), 4)
    a, b = 0.75, -2.5
    o1, _ = oracle_mod.recurrent(q, k, v1)
    o2, _ = oracle_mod.recurrent(q, k, v2)
    o12, _ = oracle_mod.recurrent(q, k, a * v1 + b * v2)
    assert _rel(o12, a * o1 + b * o2) < 1e-12
    q2 = _rand((1, N, d), 5)
    oq, _ = oracle_mod.recurrent(q2, k, v1)
    oqq, _ = oracle_mod.recurrent(a * q + b * q2, k, v1)
    assert _rel(oqq, a * o1 + b * oq) < 1e-12
    # causality: perturbing token t leaves o_{<t} untouched and changes o_t
    t = 41
    kp, vp = k.copy(), v1.copy()
    kp[0, t] += 1.0
    vp[0, t] -= 2.0
    op, _ = oracle_mod.recurrent(q, kp, vp)
    np.testing.assert_array_equal(op[0, :t], o1[0, :t])
    assert np.abs(op[0, t] - o1[0, t]).max() > 1e-3


def test_split_invariance(oracle_mod):
    """prefill(0..n) then resume(n..N) from its state equals prefill(0..N)."""
    q, k, v = synth.qkv((2, 500, 32), 32, "fp32", seed=8)
    s0 = _rand((2, 32, 32), 1)
    o, s = oracle_mod.recurrent(q, k, v, s0)
    for n in (1, 128, 333):
        oa, sa = oracle_mod.recurrent(q[:, :n], k[:, :n], v[:, :n], s0)
        ob, sb = oracle_mod.recurrent(q[:, n:], k[:, n:], v[:, n:], sa)
        assert _rel(np.concatenate([oa, ob], 1), o) < 1e-13
        assert _rel(sb, s) < 1e-13


def test_decode_matches_prefill(oracle_mod):
    q, k, v = synth.qkv((3, 4, 20, 16), 16, "fp32", seed=21)
    S0 = _rand((3, 4, 16, 16), 2)
    o, s = oracle_mod.recurrent(q, k, v, S0)
    S = S0.copy()
    for t in range(20):
        ot, S = oracle_mod.decode(q[:, :, t], k[:, :, t], v[:, :, t], S)
        assert _rel(ot, o[:, :, t]) < 1e-13
    assert _rel(S, s) < 1e-13


def test_varlen_matches_loop(oracle_mod):
    lens = [5, 0, 130, 1, 64, 77]
    H, d = 3, 8
    cu = synth.cu_seqlens(lens)
    T = int(cu[-1])
    q, k, v = synth.qkv((T, H, d), d, "fp32", seed=4)
    pool = _rand((2, H, d, d), 3)
    idx = [1, -1, 0, -1, 1, 0]
    o, s = oracle_mod.varlen(q, k, v, cu, pool, idx)
    for n, L in enumerate(lens):
        a, b = int(cu[n]), int(cu[n + 1])
        s0 = pool[idx[n]] if idx[n] >= 0 else None
        qn = q[a:b].permute(1, 0, 2)
        kn = k[a:b].permute(1, 0, 2)
        vn = v[a:b].permute(1, 0, 2)
        on, sn = oracle_mod.recurrent(qn, kn, vn, s0)
        assert np.array_equal(o[a:b], on.transpose(1, 0, 2))
        want_s = sn if L else (s0 if s0 is not None else np.zeros((H, d, d)))
        assert np.array_equal(s[n], want_s)


def test_empty_sequence(oracle_mod):
    q = np.zeros((2, 0, 8))
    s0 = _rand((2, 8, 8), 1)
    o, s = oracle_mod.recurrent(q, q, q, s0)
    assert o.shape == (2, 0, 8)
    np.testing.assert_array_equal(s, s0)


# ------------------------------------------------- planted mistakes (mutants)
def _mutant_exclusive(q, k, v, s0):
    """Wrong: o_t = q_t S_{t-1} (mask without the diagonal)."""
    S = s0.copy()
    o = np.zeros((q.shape[0], v.shape[1]))
    for t in range(q.shape[0]):
        o[t] = q[t] @ S
        S = S + np.outer(k[t], v[t])
    return o, S


def _mutant_transposed(q, k, v, s0):
    """Wrong: the state is read transposed, o_t = S_t q_t (needs dk == dv)."""
    S = s0.copy()
    o = np.zeros((q.shape[0], v.shape[1]))
    for t in range(q.shape[0]):
        S = S + np.outer(k[t], v[t])
        o[t] = S @ q[t]
    return o, S


def _mutant_dropped_s0(q, k, v, s0):
    """Wrong: the initial state is ignored in the outputs."""
    o, S = _brute(q, k, v, np.zeros_like(s0))
    return o, S + s0


def _mutant_sign(q, k, v, s0):
    o, S = _brute(q, k, v, s0)
    o[1:] -= 2 * (q[1:] @ s0)
    return o, S


@pytest.mark.parametrize("mutant", [_mutant_exclusive, _mutant_transposed, _mutant_dropped_s0, _mutant_sign])
def test_pins_reject_planted_mistakes(mutant):
    """Each planted mistake fails at least one pin: the hand-worked fixture,
    brute force with a non-zero S0, or the o_1 invariant."""
    g = _read_golden("hand_worked_n3_d2.txt")
    q, k, v = (g[x].reshape(3, 2) for x in ("q", "k", "v"))
    s0 = g["B.S0"].reshape(2, 2)
    o, s = mutant(q, k, v, s0)
    fixture_ok = np.array_equal(o.reshape(-1), g["B.o"]) and np.array_equal(s.reshape(-1), g["B.S"])
    qr, kr, vr, sr = _rand((6, 4), 1), _rand((6, 4), 2), _rand((6, 4), 3), _rand((4, 4), 4)
    om, sm = mutant(qr, kr, vr, sr)
    ob, sb = _brute(qr, kr, vr, sr)
    brute_ok = _rel(om, ob) < 1e-12 and _rel(sm, sb) < 1e-12
    assert not (fixture_ok and brute_ok)


# ------------------------------------------------- low-precision state storage
# Pins of oracle/lowp.py against the definitions of the formats and of the
# recurrence, not against itself.

def test_lowp_bf16_rounding_follows_the_format_definition():
    """bfloat16 keeps 8 significant bits; halfway cases go to the even mantissa."""
    from oracle import lowp
    x = np.array([1.0, 1 + 2**-8, 1 + 3 * 2**-8, 1 + 2**-8 + 2**-20, -(1 + 2**-8), 3.0, 255.0, 257.0, 259.0],
                 dtype=np.float32)
    want = np.array([1.0, 1.0, 1 + 2**-6, 1 + 2**-7, -1.0, 3.0, 255.0, 256.0, 260.0], dtype=np.float32)
    np.testing.assert_array_equal(lowp.round_bf16(x), want)


def test_lowp_fp16_rounding_follows_the_format_definition():
    """binary16 keeps 11 significant bits, max 65504, smallest subnormal 2^-24."""
    from oracle import lowp
    x = np.array([1 + 2**-11, 1 + 3 * 2**-11, 65504.0, 2.0**-24, 2049.0, 2051.0], dtype=np.float32)
    want = np.array([1.0, 1 + 2**-9, 65504.0, 2.0**-24, 2048.0, 2052.0], dtype=np.float32)
    np.testing.assert_array_equal(lowp.round_fp16(x), want)


def _fp8_code_values(fmt):
    """Every finite value of an 8-bit format, decoded from its bit fields:
    sign | exponent (4 or 5 bits) | mantissa (3 or 2 bits).  e4m3: bias 7, the
    code with all exponent and mantissa bits set is NaN, no infinities; e5m2:
    bias 15, exponent all ones is infinity / NaN."""
    eb, mb, bias = (4, 3, 7) if fmt == "fp8_e4m3" else (5, 2, 15)
    vals = []
    for code in range(256):
        sign = -1.0 if code >> 7 else 1.0
        ef = (code >> mb) & ((1 << eb) - 1)
        mf = code & ((1 << mb) - 1)
        if fmt == "fp8_e4m3" and ef == 15 and mf == 7:
            continue
        if fmt == "fp8_e5m2" and ef == 31:
            continue
        if ef == 0:
            v = mf * 2.0 ** (1 - bias - mb)                       # subnormal
        else:
            v = (1 + mf / 2.0 ** mb) * 2.0 ** (ef - bias)
        vals.append((sign * v, mf))
    return vals


@pytest.mark.parametrize("fmt,vmax,tiny", [("fp8_e4m3", 448.0, 2.0**-9), ("fp8_e5m2", 57344.0, 2.0**-16)])
def test_lowp_fp8_rounding_follows_the_format_definition(fmt, vmax, tiny):
    """Checked against every code of the format: representable values are kept,
    the midpoint of two neighbours goes to the one with the even mantissa field,
    values beyond the largest finite one saturate."""
    from oracle import lowp
    vals = _fp8_code_values(fmt)
    pos = sorted({v: mf for v, mf in vals if v >= 0}.items())
    values = np.array([v for v, _ in vals], dtype=np.float32)
    np.testing.assert_array_equal(lowp.round_fp8(values, fmt), values)
    assert pos[-1][0] == vmax and pos[1][0] == tiny
    lo = np.array([a for (a, _), _ in zip(pos[:-1], pos[1:])])
    hi = np.array([b for _, (b, _) in zip(pos[:-1], pos[1:])])
    even_hi = np.array([mb % 2 == 0 for _, (_, mb) in zip(pos[:-1], pos[1:])])
    mid = ((lo + hi) / 2).astype(np.float32)
    assert np.array_equal(mid.astype(np.float64), (lo + hi) / 2)   # midpoints are exact in fp32
    want = np.where(even_hi, hi, lo).astype(np.float32)
    np.testing.assert_array_equal(lowp.round_fp8(mid, fmt), want)
    np.testing.assert_array_equal(lowp.round_fp8(-mid, fmt), -want)
    # just below / above a midpoint: the nearer neighbour
    np.testing.assert_array_equal(lowp.round_fp8(np.nextafter(mid, np.float32(0)), fmt), lo.astype(np.float32))
    np.testing.assert_array_equal(lowp.round_fp8(np.nextafter(mid, np.float32(np.inf)), fmt), hi.astype(np.float32))
    big = np.array([vmax * 1.01, vmax * 4, 1e30, -1e30], dtype=np.float32)
    np.testing.assert_array_equal(lowp.round_fp8(big, fmt), np.array([vmax, vmax, vmax, -vmax], dtype=np.float32))


@pytest.mark.parametrize("fmt,dtype", [("fp8_e4m3", "float8_e4m3fn"), ("fp8_e5m2", "float8_e5m2")])
def test_lowp_fp8_rounding_matches_the_library_cast_in_range(fmt, dtype):
    """Against torch's float8 cast (round to nearest even) on values inside the
    finite range, where saturation plays no part."""
    import torch
    from oracle import lowp
    rng = np.random.default_rng(11)
    vmax = lowp.FP8[fmt][2]
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-4, 1e-2, 1.0, 30.0, vmax / 8)])
    x = x[np.abs(x) < vmax].astype(np.float32)
    want = torch.from_numpy(x).to(getattr(torch, dtype)).float().numpy()
    np.testing.assert_array_equal(lowp.round_fp8(x, fmt), want)


@pytest.mark.parametrize("fmt", ["fp32", "bf16", "fp16"])
def test_lowp_decode_is_exact_where_the_format_holds_every_value(oracle_mod, fmt):
    """Integer inputs with |S| <= 64: every product, sum and stored value is
    exact in all three formats, so 20 low-precision steps equal the fp64
    recurrence bit for bit."""
    from oracle import lowp
    rng = np.random.default_rng(3)
    U, d, T = 3, 16, 20
    q, k, v = (rng.integers(-1, 2, (T, U, d)).astype(np.float64) for _ in range(3))
    S = rng.integers(-30, 31, (U, d, d)).astype(np.float64)
    S_exact, S_low = S.copy(), S.astype(np.float32)
    for t in range(T):
        o_ref, S_exact = oracle_mod.decode(q[t], k[t], v[t], S_exact)
        o, S_low = lowp.decode_lowp(q[t], k[t], v[t], S_low, fmt)
        np.testing.assert_array_equal(o, o_ref)
        np.testing.assert_array_equal(S_low.astype(np.float64), S_exact)


def test_lowp_decode_loses_updates_below_half_an_ulp():
    """The storage effect the pages warn about, in closed form: a state entry of
    256 with updates of +0.5 never moves in bf16 (ulp 2 at 256), moves by
    exactly 0.5 per step in fp16 (ulp 0.25) and in fp32."""
    from oracle import lowp
    q = np.zeros(1)
    k, v = np.ones(1), np.full(1, 0.5)
    for fmt, want in (("bf16", 256.0), ("fp16", 261.0), ("fp32", 261.0), ("fp8_e4m3", 256.0), ("fp8_e5m2", 256.0)):
        S = np.full((1, 1), 256.0, dtype=np.float32)
        for _ in range(10):
            _, S = lowp.decode_lowp(q, k, v, S, fmt)
        assert S[0, 0] == want, (fmt, S[0, 0])
    # from 4 with +0.5 per step: e4m3 (spacing 0.5 in [4, 8), 1 in [8, 16))
    # climbs to 8, where 8.5 ties to the even 8 and stays; e5m2 (spacing 1 in
    # [4, 8)) ties 4.5 to the even 4 at once; the wider formats reach 9
    for fmt, want in (("fp8_e4m3", 8.0), ("fp8_e5m2", 4.0), ("bf16", 9.0), ("fp16", 9.0), ("fp32", 9.0)):
        S = np.full((1, 1), 4.0, dtype=np.float32)
        for _ in range(10):
            _, S = lowp.decode_lowp(q, k, v, S, fmt)
        assert S[0, 0] == want, (fmt, S[0, 0])


def test_lowp_decode_fp32_tracks_the_fp64_recurrence(oracle_mod):
    from oracle import lowp
    rng = np.random.default_rng(5)
    U, d, T = 2, 32, 50
    q, k, v = (rng.standard_normal((T, U, d)) / np.sqrt(d) for _ in range(3))
    q, k, v = (x.astype(np.float32).astype(np.float64) for x in (q, k, v))
    S = (rng.standard_normal((U, d, d))).astype(np.float32)
    S64 = S.astype(np.float64)
    for t in range(T):
        o_ref, S64 = oracle_mod.decode(q[t], k[t], v[t], S64)
        o, S = lowp.decode_lowp(q[t], k[t], v[t], S, "fp32")
    assert _rel(S.astype(np.float64), S64) < 1e-6
    assert _rel(o, o_ref) < 1e-6


# ------------------------------------------------------------- feature maps

def test_feature_maps_closed_forms(oracle_mod):
    x = np.array([-2.0, -1.0, 0.0, 0.5, 3.0])
    np.testing.assert_array_equal(oracle_mod.feature_map(x, None), x)
    np.testing.assert_allclose(oracle_mod.feature_map(x, "elu1"), [np.exp(-2.0), np.exp(-1.0), 1.0, 1.5, 4.0],
                               rtol=0, atol=1e-15)
    np.testing.assert_array_equal(oracle_mod.feature_map(x, "relu"), [0.0, 0.0, 0.0, 0.5, 3.0])


@pytest.mark.parametrize("phi", ["elu1", "relu"])
def test_feature_map_enters_only_through_q_and_k(oracle_mod, phi):
    """With phi the recurrence is the identity-phi recurrence on phi(q), phi(k);
    brute force of o_t = sum_{s<=t} (phi(q_t).phi(k_s)) v_s + phi(q_t) S0."""
    q, k, v, s0 = _rand((7, 5), 41), _rand((7, 5), 42), _rand((7, 4), 43), _rand((5, 4), 44)
    o, S = oracle_mod.recurrent(q, k, v, s0, phi=phi)
    fq, fk = oracle_mod.feature_map(q, phi), oracle_mod.feature_map(k, phi)
    ob, Sb = _brute(fq, fk, v, s0)
    assert _rel(o, ob) < 1e-12 and _rel(S, Sb) < 1e-12
    oq, Sq = oracle_mod.quadratic(q, k, v, s0, phi=phi)
    assert _rel(oq, ob) < 1e-12 and _rel(Sq, Sb) < 1e-12


# ------------------------------------------------------------------ backward

def _loss(oracle_mod, q, k, v, s0, W, Z):
    o, S = oracle_mod.recurrent(q, k, v, s0)
    return float(np.sum(o * W) + np.sum(S * Z))


def test_backward_matches_finite_differences(oracle_mod):
    """Central differences of L = <O, W> + <S_N, Z> through the forward oracle;
    dL/dO = W and dL/dS_N = Z are the backward's inputs."""
    N, dk, dv = 5, 3, 4
    q, k, v = _rand((N, dk), 51), _rand((N, dk), 52), _rand((N, dv), 53)
    s0, W, Z = _rand((dk, dv), 54), _rand((N, dv), 55), _rand((dk, dv), 56)
    dq, dk_, dv_, ds0 = oracle_mod.backward(q, k, v, W, s0, Z)
    h = 1e-6
    for x, g in ((q, dq), (k, dk_), (v, dv_), (s0, ds0)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = [q, k, v, s0]
            pos = [a is x for a in args].index(True)
            ap, am = list(args), list(args)
            ap[pos], am[pos] = xp, xm
            num[idx] = (_loss(oracle_mod, *ap, W, Z) - _loss(oracle_mod, *am, W, Z)) / (2 * h)
        assert _rel(g, num) < 1e-7


def test_backward_matches_autograd_of_the_quadratic_form(oracle_mod):
    """An independent derivation: torch autograd (float64, CPU) through the
    masked quadratic form O = (Q K^T ⊙ M) V + Q S0, S_N = S0 + K^T V."""
    import torch
    N, dk, dv = 9, 4, 5
    q, k, v = _rand((2, N, dk), 61), _rand((2, N, dk), 62), _rand((2, N, dv), 63)
    s0, W, Z = _rand((2, dk, dv), 64), _rand((2, N, dv), 65), _rand((2, dk, dv), 66)
    tq, tk, tv, ts0 = (torch.tensor(x, requires_grad=True) for x in (q, k, v, s0))
    M = torch.tril(torch.ones(N, N, dtype=torch.float64))
    O = ((tq @ tk.transpose(1, 2)) * M) @ tv + tq @ ts0
    S = ts0 + tk.transpose(1, 2) @ tv
    ((O * torch.tensor(W)).sum() + (S * torch.tensor(Z)).sum()).backward()
    dq, dk_, dv_, ds0 = oracle_mod.backward(q, k, v, W, s0, Z)
    for g, t in ((dq, tq), (dk_, tk), (dv_, tv), (ds0, ts0)):
        assert _rel(g, t.grad.numpy()) < 1e-12


def test_backward_single_token_closed_form(oracle_mod):
    """N = 1, S0 = 0: o = (q.k) v, so dq = (do.v) k, dk = (do.v) q, dv = (q.k) do."""
    q, k, v, do = _rand((1, 6), 71), _rand((1, 6), 72), _rand((1, 7), 73), _rand((1, 7), 74)
    dq, dk_, dv_, ds0 = oracle_mod.backward(q, k, v, do)
    a = float(do[0] @ v[0])
    np.testing.assert_allclose(dq[0], a * k[0], rtol=1e-13)
    np.testing.assert_allclose(dk_[0], a * q[0], rtol=1e-13)
    np.testing.assert_allclose(dv_[0], float(q[0] @ k[0]) * do[0], rtol=1e-13)
    np.testing.assert_allclose(ds0, np.outer(q[0], do[0]), rtol=1e-13)
