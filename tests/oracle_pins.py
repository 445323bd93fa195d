"""Pins of the fp64 oracle against facts that do not come from the oracle.

Each pin is a function ``pin_xxx(orc, lib)`` that raises AssertionError when
the oracle handle ``lib`` (None = the real oracle) disagrees with

  * the hand-worked golden examples (tests/golden/hand_worked.txt),
  * closed forms (N = 1, constant k and v, one-hot q -> numpy cumsum),
  * exact-integer special cases that reduce to library routines
    (numpy tril/matmul on small integers, where every sum is exact),
  * brute force in pure Python on tiny inputs,
  * identities of the method (block-size invariance, segment (LASP+)
    decomposition, packed-sequence independence, causality, state carry,
    decode after prefill),
  * for the gradients: hand-worked examples, torch autograd of the dense
    forward expression (a library routine), and Euler's identity for the
    parts of the loss linear in one argument, using the forward oracle.

The same functions run in test_oracle_pins.py (real oracle) and in
test_oracle_mutations.py (oracle copies with a planted mistake, each of which
must fail at least one pin).
"""
from __future__ import annotations

import os

import numpy as np

import la_inputs

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "hand_worked.txt")


def load_golden(path=GOLDEN):
    cases, cur = {}, None
    with open(path) as f:
        for raw in f:
            line = raw.split("#", 1)[0].strip()
            if not line:
                continue
            if line.startswith("case "):
                cur = {}
                cases[line.split()[1]] = cur
            elif line == "end":
                cur = None
            else:
                key, val = line.split(":", 1)
                if key.strip() == "cu_seqlens":
                    cur["cu_seqlens"] = np.array([int(x) for x in val.split()], dtype=np.int32)
                    continue
                mats = []
                for block in val.split("|"):
                    rows = [[float(x) for x in r.split()] for r in block.split(";") if r.strip()]
                    mats.append(np.array(rows, dtype=np.float64))
                cur[key.strip()] = mats if len(mats) > 1 else mats[0]
    return cases


def _b(x):
    """float array of bf16-exact values -> bits with an H=1 axis: [T, 1, d]."""
    x = np.asarray(x, dtype=np.float64)
    return la_inputs.bf16_exact(x)[:, None, :]


def _rand_bits(T, H, d, seed, scale=0.5):
    q, k, v = la_inputs.qkv((T, H, d), seed, scale=scale)
    return la_inputs.bits(q), la_inputs.bits(k), la_inputs.bits(v)


def _f(bits):
    return la_inputs.from_bits(bits).double().numpy()


def _rel(a, b):
    n = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (n if n > 0 else 1.0)


# --------------------------------------------------------------------------
def pin_golden(orc, lib=None):
    g = load_golden()
    c = g["single_sequence_d2"]
    cu = np.array([0, 3], np.int32)
    for form in ("recurrent", "quadratic"):
        out, st = getattr(orc, form)(_b(c["q"]), _b(c["k"]), _b(c["v"]), cu, lib=lib)
        assert np.array_equal(out[:, 0, :], c["out"]), (form, out[:, 0, :])
        assert np.array_equal(st[0, 0], c["state"]), (form, st[0, 0])
    for blk in (1, 2, 3):
        out, st = orc.blocked(_b(c["q"]), _b(c["k"]), _b(c["v"]), cu, blk, lib=lib)
        assert np.array_equal(out[:, 0, :], c["out"]), ("blocked", blk)
        assert np.array_equal(st[0, 0], c["state"]), ("blocked", blk)
    out, st = orc.segmented(_b(c["q"]), _b(c["k"]), _b(c["v"]), cu, 2, 1, lib=lib)
    assert np.array_equal(out[:, 0, :], c["out"]) and np.array_equal(st[0, 0], c["state"])

    c = g["carried_state_d2"]
    sin = c["state_in"][None, None]
    for form in ("recurrent", "quadratic"):
        out, st = getattr(orc, form)(_b(c["q"]), _b(c["k"]), _b(c["v"]), cu, state_in=sin, lib=lib)
        assert np.array_equal(out[:, 0, :], c["out"]), (form, out[:, 0, :])
        assert np.array_equal(st[0, 0], c["state"]), (form, st[0, 0])
    out, st = orc.blocked(_b(c["q"]), _b(c["k"]), _b(c["v"]), cu, 2, state_in=sin, lib=lib)
    assert np.array_equal(out[:, 0, :], c["out"]) and np.array_equal(st[0, 0], c["state"])
    out, st = orc.segmented(_b(c["q"]), _b(c["k"]), _b(c["v"]), cu, 1, 1, state_in=sin, lib=lib)
    assert np.array_equal(out[:, 0, :], c["out"]) and np.array_equal(st[0, 0], c["state"])

    c = g["two_packed_sequences_d2"]
    for form in ("recurrent", "quadratic"):
        out, st = getattr(orc, form)(_b(c["q"]), _b(c["k"]), _b(c["v"]), c["cu_seqlens"], lib=lib)
        assert np.array_equal(out[:, 0, :], c["out"]), form
        assert np.array_equal(st[0, 0], c["state"][0]) and np.array_equal(st[1, 0], c["state"][1]), form

    c = g["decode_after_single_sequence_d2"]
    b1 = lambda x: la_inputs.bf16_exact(np.asarray(x, np.float64).reshape(1, 1, -1))  # noqa: E731
    out, st = orc.decode_step(b1(c["q"]), b1(c["k"]), b1(c["v"]),
                              c["state_in"].reshape(1, 1, 2, 2), lib=lib)
    assert np.array_equal(out.reshape(-1), c["out"].reshape(-1)), out
    assert np.array_equal(st.reshape(2, 2), c["state"]), st


def pin_single_token(orc, lib=None):
    """N = 1: o_1 = (q_1 . k_1) v_1 and S = k_1^T v_1 (numpy dot / outer)."""
    Q, K, V = _rand_bits(1, 3, 8, seed=11)
    cu = np.array([0, 1], np.int32)
    q, k, v = _f(Q), _f(K), _f(V)
    for form in ("recurrent", "quadratic"):
        out, st = getattr(orc, form)(Q, K, V, cu, lib=lib)
        for h in range(3):
            exp = np.dot(q[0, h], k[0, h]) * v[0, h]
            assert np.allclose(out[0, h], exp, rtol=1e-14, atol=1e-300), form
            assert np.allclose(st[0, h], np.outer(k[0, h], v[0, h]), rtol=1e-14, atol=1e-300)


def pin_constant_kv(orc, lib=None):
    """k_t = k, v_t = v for all t: o_t = (t+1) (q_t . k) v  (t counted from 0)."""
    T, d = 37, 8
    Q, K, V = _rand_bits(T, 1, d, seed=12)
    K[:] = K[0]
    V[:] = V[0]
    cu = np.array([0, T], np.int32)
    q, k, v = _f(Q), _f(K), _f(V)
    for form in ("recurrent", "quadratic"):
        out, st = getattr(orc, form)(Q, K, V, cu, lib=lib)
        for t in range(T):
            exp = (t + 1) * np.dot(q[t, 0], k[0, 0]) * v[0, 0]
            assert np.allclose(out[t, 0], exp, rtol=1e-12, atol=1e-14), (form, t)
        assert np.allclose(st[0, 0], T * np.outer(k[0, 0], v[0, 0]), rtol=1e-12)
    out, _ = orc.blocked(Q, K, V, cu, 8, lib=lib)
    for t in range(T):
        assert np.allclose(out[t, 0], (t + 1) * np.dot(q[t, 0], k[0, 0]) * v[0, 0], rtol=1e-12, atol=1e-14)


def pin_one_hot_q(orc, lib=None):
    """q_t = e_i: o_t = sum_{s<=t} k_s[i] v_s = numpy cumsum over s of k_s[i] v_s."""
    T, d = 29, 6
    Q, K, V = _rand_bits(T, 1, d, seed=13)
    cu = np.array([0, T], np.int32)
    k, v = _f(K)[:, 0], _f(V)[:, 0]
    for i in (0, 3, d - 1):
        onehot = np.zeros((T, 1, d))
        onehot[:, 0, i] = 1.0
        Qi = la_inputs.bf16_exact(onehot)
        exp = np.cumsum(k[:, i:i + 1] * v, axis=0)
        for form in ("recurrent", "quadratic"):
            out, _ = getattr(orc, form)(Qi, K, V, cu, lib=lib)
            assert np.allclose(out[:, 0], exp, rtol=1e-12, atol=1e-14), (form, i)
        out, _ = orc.blocked(Qi, K, V, cu, 4, lib=lib)
        assert np.allclose(out[:, 0], exp, rtol=1e-12, atol=1e-14)


def pin_exact_integers(orc, lib=None):
    """Small-integer inputs: every sum is exact, so the oracle must equal
    numpy's tril(Q K^T) @ V and K^T V bit for bit (two packed sequences)."""
    rng = np.random.default_rng(14)
    lens = [13, 22]
    T, H, d = sum(lens), 2, 5
    qf = rng.integers(-3, 4, (T, H, d)).astype(np.float64)
    kf = rng.integers(-3, 4, (T, H, d)).astype(np.float64)
    vf = rng.integers(-3, 4, (T, H, d)).astype(np.float64)
    sin = rng.integers(-2, 3, (2, H, d, d)).astype(np.float64)
    Q, K, V = la_inputs.bf16_exact(qf), la_inputs.bf16_exact(kf), la_inputs.bf16_exact(vf)
    cu = la_inputs.cu_seqlens_from_lengths(lens)
    exp_out = np.zeros((T, H, d))
    exp_st = np.zeros((2, H, d, d))
    for i in range(2):
        a, b = cu[i], cu[i + 1]
        for h in range(H):
            qs, ks, vs = qf[a:b, h], kf[a:b, h], vf[a:b, h]
            exp_out[a:b, h] = np.tril(qs @ ks.T) @ vs + qs @ sin[i, h]
            exp_st[i, h] = sin[i, h] + ks.T @ vs
    runs = {
        "recurrent": orc.recurrent(Q, K, V, cu, state_in=sin, lib=lib),
        "quadratic": orc.quadratic(Q, K, V, cu, state_in=sin, lib=lib),
        "blocked4": orc.blocked(Q, K, V, cu, 4, state_in=sin, lib=lib),
        "segmented": orc.segmented(Q, K, V, cu, 6, 4, state_in=sin, lib=lib),
    }
    for name, (out, st) in runs.items():
        assert np.array_equal(out, exp_out), name
        assert np.array_equal(st, exp_st), name
    # a subset of heads, in a different order, gives the same rows
    out, st = orc.recurrent(Q, K, V, cu, heads=[1, 0], state_in=sin[:, ::-1], lib=lib)
    assert np.array_equal(out, exp_out[:, ::-1]) and np.array_equal(st, exp_st[:, ::-1])


def pin_brute_force(orc, lib=None):
    """Pure-Python sums over (t, s, a, b) on tiny inputs, several d."""
    for seed, (T, d) in enumerate([(1, 1), (5, 2), (8, 3), (7, 4)]):
        Q, K, V = _rand_bits(T, 1, d, seed=100 + seed)
        q, k, v = _f(Q)[:, 0].tolist(), _f(K)[:, 0].tolist(), _f(V)[:, 0].tolist()
        exp = [[sum(sum(q[t][a] * k[s][a] for a in range(d)) * v[s][b] for s in range(t + 1))
                for b in range(d)] for t in range(T)]
        st = [[sum(k[s][a] * v[s][b] for s in range(T)) for b in range(d)] for a in range(d)]
        cu = np.array([0, T], np.int32)
        for form in ("recurrent", "quadratic"):
            out, so = getattr(orc, form)(Q, K, V, cu, lib=lib)
            assert np.allclose(out[:, 0], np.array(exp), rtol=1e-12, atol=1e-15), (form, T, d)
            assert np.allclose(so[0, 0], np.array(st), rtol=1e-12, atol=1e-15), (form, T, d)


def pin_forms_agree(orc, lib=None):
    """recurrent == quadratic == blocked(every block size) == segmented."""
    T, H, d = 64, 2, 8
    Q, K, V = _rand_bits(T, H, d, seed=15)
    cu = np.array([0, T], np.int32)
    sin = np.random.default_rng(5).normal(size=(1, H, d, d))
    ref, rst = orc.quadratic(Q, K, V, cu, state_in=sin, lib=lib)
    out, st = orc.recurrent(Q, K, V, cu, state_in=sin, lib=lib)
    assert _rel(out, ref) < 1e-12 and _rel(st, rst) < 1e-12
    for blk in range(1, T + 1):
        out, st = orc.blocked(Q, K, V, cu, blk, state_in=sin, lib=lib)
        assert _rel(out, ref) < 1e-12 and _rel(st, rst) < 1e-12, blk
    for seg, blk in [(1, 1), (16, 8), (24, 5), (64, 64), (100, 7)]:
        out, st = orc.segmented(Q, K, V, cu, seg, blk, state_in=sin, lib=lib)
        assert _rel(out, ref) < 1e-12 and _rel(st, rst) < 1e-12, (seg, blk)


def pin_causality_and_packing(orc, lib=None):
    """Changing future tokens leaves earlier outputs bit-identical; changing
    one packed sequence leaves every other sequence bit-identical."""
    lens = [9, 1, 17, 0, 12]
    T, H, d = sum(lens), 2, 4
    Q, K, V = _rand_bits(T, H, d, seed=16)
    cu = la_inputs.cu_seqlens_from_lengths(lens)
    base, bst = orc.recurrent(Q, K, V, cu, lib=lib)
    t_cut = 5
    Q2, K2, V2 = Q.copy(), K.copy(), V.copy()
    Q2[t_cut + 1:], K2[t_cut + 1:], V2[t_cut + 1:] = _rand_bits(T - t_cut - 1, H, d, seed=17)
    out, _ = orc.recurrent(Q2, K2, V2, cu, lib=lib)
    assert np.array_equal(out[:t_cut + 1], base[:t_cut + 1])
    assert not np.array_equal(out[t_cut + 1:cu[1]], base[t_cut + 1:cu[1]])
    a, b = cu[2], cu[3]                       # perturb sequence 2 only
    Q3, K3, V3 = Q.copy(), K.copy(), V.copy()
    Q3[a:b], K3[a:b], V3[a:b] = _rand_bits(b - a, H, d, seed=18)
    for form in ("recurrent", "quadratic"):
        out, st = getattr(orc, form)(Q3, K3, V3, cu, lib=lib)
        ref, rst = (base, bst) if form == "recurrent" else orc.quadratic(Q, K, V, cu, lib=lib)
        assert np.array_equal(out[:a], ref[:a]) and np.array_equal(out[b:], ref[b:]), form
        for i in (0, 1, 3, 4):
            assert np.array_equal(st[i], rst[i]), (form, i)
        assert not np.allclose(out[a:b], ref[a:b])
    # a zero-length sequence keeps its carried-in state and emits nothing
    sin = np.random.default_rng(6).normal(size=(len(lens), H, d, d))
    _, st = orc.recurrent(Q, K, V, cu, state_in=sin, lib=lib)
    assert np.array_equal(st[3], sin[3])


def pin_state_carry_and_decode(orc, lib=None):
    """prefill(A) then prefill(B, S_A) == prefill(A ++ B); prefill(N) followed
    by m decode steps == prefill(N + m) (outputs of the last m tokens, state)."""
    N, m, H, d = 40, 6, 3, 8
    Q, K, V = _rand_bits(N + m, H, d, seed=19)
    full, fst = orc.recurrent(Q, K, V, np.array([0, N + m], np.int32), lib=lib)
    fq, fqs = orc.quadratic(Q, K, V, np.array([0, N + m], np.int32), lib=lib)
    assert _rel(full, fq) < 1e-12 and _rel(fst, fqs) < 1e-12
    _, sA = orc.recurrent(Q[:N], K[:N], V[:N], np.array([0, N], np.int32), lib=lib)
    outB, sB = orc.quadratic(Q[N:], K[N:], V[N:], np.array([0, m], np.int32), state_in=sA, lib=lib)
    assert _rel(outB, full[N:]) < 1e-12 and _rel(sB, fst) < 1e-12
    state = sA[0][None]                                   # [1, H, d, d]
    for t in range(N, N + m):
        o, state = orc.decode_step(Q[t][None], K[t][None], V[t][None], state, lib=lib)
        assert _rel(o[0], full[t]) < 1e-12, t
    assert _rel(state[0], fst[0]) < 1e-12


def pin_linearity(orc, lib=None):
    """O is linear in V (2V -> 2O exactly: scaling by 2 is exact in bf16 and fp64)
    and bilinear in (Q, K) the same way; negating V negates O and S."""
    T, H, d = 33, 1, 6
    Q, K, V = _rand_bits(T, H, d, seed=20)
    cu = np.array([0, T], np.int32)
    two = lambda b: la_inputs.bf16_exact(2.0 * _f(b))       # noqa: E731
    neg = lambda b: la_inputs.bf16_exact(-_f(b))            # noqa: E731
    o, s = orc.recurrent(Q, K, V, cu, lib=lib)
    o2, s2 = orc.recurrent(Q, K, two(V), cu, lib=lib)
    assert np.array_equal(o2, 2 * o) and np.array_equal(s2, 2 * s)
    o3, s3 = orc.quadratic(two(Q), K, V, cu, lib=lib)
    assert _rel(o3, 2 * o) < 1e-13 and _rel(s3, s) < 1e-13
    o4, s4 = orc.recurrent(Q, K, neg(V), cu, lib=lib)
    assert np.array_equal(o4, -o) and np.array_equal(s4, -s)


# -------------------------------------------------------------------------- gradients
def pin_backward_golden(orc, lib=None):
    """The hand-worked gradient examples (d = 1 and d = 2), exact."""
    g = load_golden()
    for name in ("backward_d1", "backward_d2"):
        c = g[name]
        d = c["q"].shape[1]
        cu = np.array([0, c["q"].shape[0]], np.int32)
        dq, dk, dv, dsin = orc.backward(_b(c["q"]), _b(c["k"]), _b(c["v"]), _b(c["dout"]), cu,
                                        state_in=c["state_in"].reshape(1, 1, d, d),
                                        dstate_out=c["dstate_out"].reshape(1, 1, d, d), lib=lib)
        assert np.array_equal(dq[:, 0], c["dq"]), (name, "dq", dq[:, 0])
        assert np.array_equal(dk[:, 0], c["dk"]), (name, "dk", dk[:, 0])
        assert np.array_equal(dv[:, 0], c["dv"]), (name, "dv", dv[:, 0])
        assert np.array_equal(dsin[0, 0], c["dstate_in"]), (name, "dS_in", dsin[0, 0])


def _autograd_reference(Qf, Kf, Vf, Gf, cu, Sin, GS):
    """torch autograd (a library routine) of the dense forward expression, one
    sequence at a time, in fp64."""
    import torch
    outs = [np.zeros_like(Qf) for _ in range(3)]
    dsin = np.zeros_like(Sin)
    for i in range(len(cu) - 1):
        a, b = int(cu[i]), int(cu[i + 1])
        for h in range(Qf.shape[1]):
            q, k, v = (torch.tensor(x[a:b, h], dtype=torch.float64, requires_grad=True) for x in (Qf, Kf, Vf))
            s_in = torch.tensor(Sin[i, h], dtype=torch.float64, requires_grad=True)
            o = torch.tril(q @ k.T) @ v + q @ s_in
            s_out = s_in + k.T @ v
            loss = (torch.tensor(Gf[a:b, h]) * o).sum() + (torch.tensor(GS[i, h]) * s_out).sum()
            loss.backward()
            for dst, x in zip(outs, (q, k, v)):
                dst[a:b, h] = x.grad.numpy()
            dsin[i, h] = s_in.grad.numpy()
    return outs + [dsin]


def pin_backward_autograd(orc, lib=None):
    """Packed sequences (one empty) with carried-in states and state
    gradients: the oracle's gradients equal torch autograd's to rounding."""
    H, d = 2, 5
    cu = np.array([0, 7, 7, 30, 41], np.int32)
    T = int(cu[-1])
    Q, K, V = _rand_bits(T, H, d, seed=31)
    G, _, _ = _rand_bits(T, H, d, seed=32)
    rng = np.random.default_rng(33)
    Sin = rng.standard_normal((4, H, d, d))
    GS = rng.standard_normal((4, H, d, d))
    got = orc.backward(Q, K, V, G, cu, state_in=Sin, dstate_out=GS, lib=lib)
    ref = _autograd_reference(_f(Q), _f(K), _f(V), _f(G), cu, Sin, GS)
    for name, x, y in zip(("dq", "dk", "dv", "dS_in"), got, ref):
        assert _rel(x, y) < 1e-12, (name, _rel(x, y))
    # without carried-in state and state gradient: the same as zeros
    got0 = orc.backward(Q, K, V, G, cu, lib=lib)
    ref0 = _autograd_reference(_f(Q), _f(K), _f(V), _f(G), cu, np.zeros_like(Sin), np.zeros_like(GS))
    for x, y in zip(got0, ref0):
        assert _rel(x, y) < 1e-12


def pin_backward_homogeneity(orc, lib=None):
    """Euler's identity for the pieces of the loss L = <g, o> + <G, S_out>
    that are linear in one argument, with o and S_out from the (separately
    pinned) forward oracle:
      sum q.dq = <g, o>;   sum k.dk = sum v.dv = <g, o_intra> + <G, S_out - S_in>;
      <S_in, dS_in> = <g, o - o_intra> + <G, S_in>."""
    H, d = 1, 6
    cu = np.array([0, 19, 40], np.int32)
    T = int(cu[-1])
    Q, K, V = _rand_bits(T, H, d, seed=35)
    G, _, _ = _rand_bits(T, H, d, seed=36)
    rng = np.random.default_rng(37)
    Sin = rng.standard_normal((2, H, d, d))
    GS = rng.standard_normal((2, H, d, d))
    dq, dk, dv, dsin = orc.backward(Q, K, V, G, cu, state_in=Sin, dstate_out=GS, lib=lib)
    o, s_out = orc.quadratic(Q, K, V, cu, state_in=Sin, lib=lib)
    o_intra, kv = orc.quadratic(Q, K, V, cu, lib=lib)
    g = _f(G)
    L_o, L_intra = float((g * o).sum()), float((g * o_intra).sum())
    assert abs(float((_f(Q) * dq).sum()) - L_o) < 1e-11 * max(1.0, abs(L_o))
    rhs = L_intra + float((GS * kv).sum())
    for x, dx in ((_f(K), dk), (_f(V), dv)):
        assert abs(float((x * dx).sum()) - rhs) < 1e-11 * max(1.0, abs(rhs))
    rhs_s = (L_o - L_intra) + float((GS * Sin).sum())
    assert abs(float((Sin * dsin).sum()) - rhs_s) < 1e-11 * max(1.0, abs(rhs_s))
    assert np.allclose(s_out - Sin, kv, rtol=0, atol=1e-12)


# -------------------------------------------------------------------------- per-head decay
def _decays(H, seed):
    """Per-head decays in (0, 1], one exactly 1 and one small."""
    lam = np.random.default_rng(seed).uniform(0.55, 0.999, H)
    lam[0] = 1.0
    if H > 2:
        lam[-1] = 0.2
    return lam


def pin_decay_one_is_undecayed(orc, lib=None):
    """lambda = 1 on every head: each decayed form equals its undecayed
    counterpart bit for bit (every extra factor is an exact 1.0)."""
    lens = [11, 0, 23, 6]
    T, H, d = sum(lens), 3, 5
    Q, K, V = _rand_bits(T, H, d, seed=40)
    cu = la_inputs.cu_seqlens_from_lengths(lens)
    sin = np.random.default_rng(41).normal(size=(len(lens), H, d, d))
    one = np.ones(H)
    pairs = [
        (orc.recurrent_decay(Q, K, V, cu, one, state_in=sin, lib=lib), orc.recurrent(Q, K, V, cu, state_in=sin, lib=lib)),
        (orc.quadratic_decay(Q, K, V, cu, one, state_in=sin, lib=lib), orc.quadratic(Q, K, V, cu, state_in=sin, lib=lib)),
        (orc.blocked_decay(Q, K, V, cu, 4, one, state_in=sin, lib=lib),
         orc.blocked(Q, K, V, cu, 4, state_in=sin, lib=lib)),
        (orc.segmented_decay(Q, K, V, cu, 8, 3, one, state_in=sin, lib=lib),
         orc.segmented(Q, K, V, cu, 8, 3, state_in=sin, lib=lib)),
    ]
    for i, ((o1, s1), (o2, s2)) in enumerate(pairs):
        assert np.array_equal(o1, o2) and np.array_equal(s1, s2), i
    Qd, Kd, Vd = _rand_bits(2 * H, 1, d, seed=42)
    sd = np.random.default_rng(43).normal(size=(2, H, d, d))
    shp = lambda x: x.reshape(2, H, d)  # noqa: E731
    o1, s1 = orc.decode_step_decay(shp(Qd), shp(Kd), shp(Vd), sd, one, lib=lib)
    o2, s2 = orc.decode_step(shp(Qd), shp(Kd), shp(Vd), sd, lib=lib)
    assert np.array_equal(o1, o2) and np.array_equal(s1, s2)


def pin_decay_brute_force(orc, lib=None):
    """Pure-Python sums o_t[b] = sum_{s<=t} lam^(t-s) sum_a q_t[a] k_s[a] v_s[b]
    + lam^(t+1) sum_a q_t[a] S_in[a][b] and the final state, tiny inputs."""
    for seed, (T, d, lam) in enumerate([(1, 1, 0.5), (6, 2, 0.9), (9, 3, 0.3), (7, 4, 0.77)]):
        Q, K, V = _rand_bits(T, 1, d, seed=110 + seed)
        sin = np.random.default_rng(120 + seed).normal(size=(1, 1, d, d))
        q, k, v, S = _f(Q)[:, 0].tolist(), _f(K)[:, 0].tolist(), _f(V)[:, 0].tolist(), sin[0, 0].tolist()
        exp = [[sum(lam ** (t - s) * sum(q[t][a] * k[s][a] for a in range(d)) * v[s][b] for s in range(t + 1))
                + lam ** (t + 1) * sum(q[t][a] * S[a][b] for a in range(d))
                for b in range(d)] for t in range(T)]
        st = [[lam ** T * S[a][b] + sum(lam ** (T - 1 - s) * k[s][a] * v[s][b] for s in range(T))
               for b in range(d)] for a in range(d)]
        cu = np.array([0, T], np.int32)
        for form in ("recurrent_decay", "quadratic_decay"):
            out, so = getattr(orc, form)(Q, K, V, cu, [lam], state_in=sin, lib=lib)
            assert np.allclose(out[:, 0], np.array(exp), rtol=1e-12, atol=1e-15), (form, T, d)
            assert np.allclose(so[0, 0], np.array(st), rtol=1e-12, atol=1e-15), (form, T, d)


def pin_decay_constant_kv(orc, lib=None):
    """k_t = k, v_t = v: S_t = lam^(t+1) S_in + (1 - lam^(t+1)) / (1 - lam) k^T v
    (a geometric series), o_t = q_t S_t."""
    T, d, H = 41, 6, 2
    Q, K, V = _rand_bits(T, H, d, seed=44)
    K[:] = K[0]
    V[:] = V[0]
    lam = np.array([0.93, 0.6])
    sin = np.random.default_rng(45).normal(size=(1, H, d, d))
    cu = np.array([0, T], np.int32)
    q, k, v = _f(Q), _f(K), _f(V)
    for form in ("recurrent_decay", "quadratic_decay"):
        out, st = getattr(orc, form)(Q, K, V, cu, lam, state_in=sin, lib=lib)
        for h in range(H):
            kv = np.outer(k[0, h], v[0, h])
            for t in range(T):
                S_t = lam[h] ** (t + 1) * sin[0, h] + (1 - lam[h] ** (t + 1)) / (1 - lam[h]) * kv
                assert np.allclose(out[t, h], q[t, h] @ S_t, rtol=1e-11, atol=1e-13), (form, h, t)
            S_T = lam[h] ** T * sin[0, h] + (1 - lam[h] ** T) / (1 - lam[h]) * kv
            assert np.allclose(st[0, h], S_T, rtol=1e-11, atol=1e-13), (form, h)


def pin_decay_exact_half(orc, lib=None):
    """lam = 1/2 (an exact power of two) and small-integer inputs: every term
    is exact, so the oracle must equal numpy's ((Q K^T) ⊙ D) V + diag(2^-(t+1)) Q S_in
    with D[t][s] = 2^-(t-s) for s <= t, and the matching final state, bit for bit."""
    rng = np.random.default_rng(46)
    lens = [12, 9]
    T, H, d = sum(lens), 2, 4
    qf = rng.integers(-3, 4, (T, H, d)).astype(np.float64)
    kf = rng.integers(-3, 4, (T, H, d)).astype(np.float64)
    vf = rng.integers(-3, 4, (T, H, d)).astype(np.float64)
    sin = rng.integers(-2, 3, (2, H, d, d)).astype(np.float64)
    Q, K, V = la_inputs.bf16_exact(qf), la_inputs.bf16_exact(kf), la_inputs.bf16_exact(vf)
    cu = la_inputs.cu_seqlens_from_lengths(lens)
    lam = np.array([0.5, 1.0])
    exp_out = np.zeros((T, H, d))
    exp_st = np.zeros((2, H, d, d))
    for i in range(2):
        a, b = cu[i], cu[i + 1]
        n = b - a
        for h in range(H):
            tt = np.arange(n)
            D = np.tril(lam[h] ** (tt[:, None] - tt[None, :]).clip(min=0))
            qs, ks, vs = qf[a:b, h], kf[a:b, h], vf[a:b, h]
            exp_out[a:b, h] = ((qs @ ks.T) * D) @ vs + (lam[h] ** (tt + 1))[:, None] * (qs @ sin[i, h])
            exp_st[i, h] = lam[h] ** n * sin[i, h] + (ks * (lam[h] ** (n - 1 - tt))[:, None]).T @ vs
    runs = {
        "recurrent": orc.recurrent_decay(Q, K, V, cu, lam, state_in=sin, lib=lib),
        "quadratic": orc.quadratic_decay(Q, K, V, cu, lam, state_in=sin, lib=lib),
        "blocked5": orc.blocked_decay(Q, K, V, cu, 5, lam, state_in=sin, lib=lib),
        "segmented": orc.segmented_decay(Q, K, V, cu, 7, 3, lam, state_in=sin, lib=lib),
    }
    for name, (out, st) in runs.items():
        assert np.array_equal(out, exp_out), name
        assert np.array_equal(st, exp_st), name


def pin_decay_forms_agree(orc, lib=None):
    """recurrent == quadratic == blocked (every block size) == segmented under
    decay, with packed sequences and a carried-in state; lam -> 0 leaves only
    the diagonal term (q_t . k_t) v_t."""
    lens = [37, 27]
    T, H, d = sum(lens), 3, 6
    Q, K, V = _rand_bits(T, H, d, seed=47)
    cu = la_inputs.cu_seqlens_from_lengths(lens)
    lam = _decays(H, 48)
    sin = np.random.default_rng(49).normal(size=(2, H, d, d))
    ref, rst = orc.quadratic_decay(Q, K, V, cu, lam, state_in=sin, lib=lib)
    out, st = orc.recurrent_decay(Q, K, V, cu, lam, state_in=sin, lib=lib)
    assert _rel(out, ref) < 1e-12 and _rel(st, rst) < 1e-12
    for blk in range(1, max(lens) + 1):
        out, st = orc.blocked_decay(Q, K, V, cu, blk, lam, state_in=sin, lib=lib)
        assert _rel(out, ref) < 1e-12 and _rel(st, rst) < 1e-12, blk
    for seg, blk in [(1, 1), (8, 4), (10, 3), (37, 37), (50, 6)]:
        out, st = orc.segmented_decay(Q, K, V, cu, seg, blk, lam, state_in=sin, lib=lib)
        assert _rel(out, ref) < 1e-12 and _rel(st, rst) < 1e-12, (seg, blk)
    zero = np.zeros(H)
    q, k, v = _f(Q), _f(K), _f(V)
    exp = np.einsum("tha,tha->th", q, k)[:, :, None] * v
    for form in ("recurrent_decay", "quadratic_decay"):
        out, st = getattr(orc, form)(Q, K, V, cu, zero, state_in=sin, lib=lib)
        assert np.allclose(out, exp, rtol=1e-14, atol=1e-300), form
        for i in range(2):
            last = cu[i + 1] - 1
            assert np.allclose(st[i], np.einsum("ha,hb->hab", k[last], v[last]), rtol=1e-14, atol=1e-300)


def pin_decay_carry_and_decode(orc, lib=None):
    """prefill(A) then prefill(B, S_A) == prefill(A ++ B) and prefill(N) then m
    decayed decode steps == prefill(N + m), with per-head decays."""
    N, m, H, d = 30, 5, 3, 6
    Q, K, V = _rand_bits(N + m, H, d, seed=50)
    lam = _decays(H, 51)
    full, fst = orc.recurrent_decay(Q, K, V, np.array([0, N + m], np.int32), lam, lib=lib)
    _, sA = orc.quadratic_decay(Q[:N], K[:N], V[:N], np.array([0, N], np.int32), lam, lib=lib)
    outB, sB = orc.blocked_decay(Q[N:], K[N:], V[N:], np.array([0, m], np.int32), 2, lam, state_in=sA, lib=lib)
    assert _rel(outB, full[N:]) < 1e-12 and _rel(sB, fst) < 1e-12
    state = sA[0][None]
    for t in range(N, N + m):
        o, state = orc.decode_step_decay(Q[t][None], K[t][None], V[t][None], state, lam, lib=lib)
        assert _rel(o[0], full[t]) < 1e-12, t
    assert _rel(state[0], fst[0]) < 1e-12
    # a subset of heads, in another order, reads the decay of its own head number
    out, st = orc.recurrent_decay(Q, K, V, np.array([0, N + m], np.int32), lam, heads=[2, 0], lib=lib)
    assert np.array_equal(out, full[:, [2, 0]]) and np.array_equal(st, fst[:, [2, 0]])


ALL_PINS = [pin_golden, pin_single_token, pin_constant_kv, pin_one_hot_q, pin_exact_integers,
            pin_brute_force, pin_forms_agree, pin_causality_and_packing,
            pin_state_carry_and_decode, pin_linearity, pin_backward_golden, pin_backward_autograd,
            pin_backward_homogeneity, pin_decay_one_is_undecayed, pin_decay_brute_force,
            pin_decay_constant_kv, pin_decay_exact_half, pin_decay_forms_agree, pin_decay_carry_and_decode]
