"""Pins of the oracle's 3D rotary position encoding (CPU).

The pages name the method (video / 3D RoPE on Q and K, a timestamp on the
summary tokens) but print no formula; the oracle restates RoFormer's rotary
encoding (Su et al. 2021) over three axes (time, patch row, patch column) with
the 64 head dims split 24/20/20.  These tests pin it to what rotary encoding
must satisfy, independently of how the oracle builds its matrices:
the identity at position 0, orthogonality, scores that depend on positions
only through their differences (per axis and jointly, against the complex-number
closed form), the dims each axis owns, and GCA outputs that do not move when
every frame's timestamp is shifted by the same amount.
"""
import math

import numpy as np
import pytest

from oracle import gca

D = 64


def _rng(seed=0):
    return np.random.default_rng(seed)


def test_position_zero_is_the_identity():
    assert np.array_equal(gca.rope_matrix(0, 0, 0), np.eye(D))


@pytest.mark.parametrize("pos", [(1, 0, 0), (0, 3, 0), (0, 0, 7), (9999, 26, 36), (0.5, 1.5, 2.5)])
def test_rotation_is_orthogonal_and_keeps_norms(pos):
    R = gca.rope_matrix(*pos)
    assert np.abs(R @ R.T - np.eye(D)).max() < 1e-12
    assert abs(np.linalg.det(R) - 1.0) < 1e-9
    x = _rng(1).standard_normal(D)
    assert abs(np.linalg.norm(R @ x) - np.linalg.norm(x)) < 1e-12


def test_each_axis_owns_its_dims():
    # time rotates dims 0..23, patch row dims 24..43, patch column dims 44..63
    for pos, lo, hi in (((5, 0, 0), 0, 24), ((0, 5, 0), 24, 44), ((0, 0, 5), 44, 64)):
        R = gca.rope_matrix(*pos)
        rest = [d for d in range(D) if not lo <= d < hi]
        assert np.array_equal(R[np.ix_(rest, rest)], np.eye(len(rest)))
        assert np.abs(R[lo:hi, lo:hi] - np.eye(hi - lo)).max() > 0.1


def _complex_score(q, k, pq, pk):
    """<R(pq) q, R(pk) k> from the closed form: pair i of q and k as complex
    numbers, Re(q_i * conj(k_i) * exp(i (a_i(pq) - a_i(pk))))."""
    qc = q[0::2] + 1j * q[1::2]
    kc = k[0::2] + 1j * k[1::2]
    da = gca.rope_angles(*pq) - gca.rope_angles(*pk)
    return float(np.real(np.sum(qc * np.conj(kc) * np.exp(1j * da))))


def test_pair_rotation_is_multiplication_by_exp_i_angle():
    x = _rng(2).standard_normal(D)
    pos = (17, 4, 11)
    y = gca.rope_matrix(*pos) @ x
    xc = x[0::2] + 1j * x[1::2]
    yc = y[0::2] + 1j * y[1::2]
    assert np.abs(yc - xc * np.exp(1j * gca.rope_angles(*pos))).max() < 1e-12
    # the first pair of every axis turns by exactly one radian per position step
    a = gca.rope_angles(3, 5, 7)
    assert (a[0], a[12], a[22]) == (3.0, 5.0, 7.0)


def test_scores_depend_only_on_position_differences():
    rng = _rng(3)
    for _ in range(20):
        q, k = rng.standard_normal(D), rng.standard_normal(D)
        pq = tuple(rng.integers(0, 10000, 1)[0] if a == 0 else rng.integers(0, 40, 1)[0] for a in range(3))
        pk = tuple(rng.integers(0, 10000, 1)[0] if a == 0 else rng.integers(0, 40, 1)[0] for a in range(3))
        shift = tuple(rng.integers(-50, 50, 3))
        s0 = (gca.rope_matrix(*pq) @ q) @ (gca.rope_matrix(*pk) @ k)
        s1 = (gca.rope_matrix(*[a + b for a, b in zip(pq, shift)]) @ q) @ \
             (gca.rope_matrix(*[a + b for a, b in zip(pk, shift)]) @ k)
        assert abs(s0 - s1) < 1e-9 * (1 + abs(s0))
        assert abs(s0 - _complex_score(q, k, pq, pk)) < 1e-9 * (1 + abs(s0))


def test_token_positions_follow_the_patch_grid():
    # 518x378 at patch 14: a 37-wide, 27-high grid, special tokens first
    pos = gca.token_positions(42, 6, 999, 37)
    assert pos[:6] == [(42, 0, 0)] * 6
    assert pos[6] == (42, 0, 0) and pos[6 + 36] == (42, 0, 36) and pos[6 + 37] == (42, 1, 0)
    assert pos[-1] == (42, 26, 36)


def test_bf16_rounding_matches_torch():
    import torch
    x = _rng(4).standard_normal(10000) * 10.0 ** _rng(5).integers(-5, 5, 10000)
    x32 = x.astype(np.float32)
    got = gca.round_to_dtype(x32, "bf16")
    want = torch.from_numpy(x32).to(torch.bfloat16).double().numpy()
    assert np.array_equal(got, want)


def _rope_stream(T, shift, dtype="f32", seed=0, rope=True):
    """A small GCA stream whose K and Q are rotated with timestamps frame+shift
    (or left unrotated with rope=False)."""
    M, S, H, n, k, gw = 12, 6, 2, 2, 3, 4
    rng = _rng(seed)
    Q = rng.standard_normal((T, S + M, H, D)).astype(np.float32)
    K = rng.standard_normal((T, S + M, H, D)).astype(np.float32)
    V = rng.standard_normal((T, S + M, H, D)).astype(np.float32)
    rot = (lambda x, t: gca.rope_frame(x, t + shift, S=S, grid_w=gw, dtype=dtype)) if rope else \
        (lambda x, t: x)
    Kr = {t: rot(K[t], t) for t in range(T)}

    def fkv(j, summary_only):
        return (Kr[j][:S], V[j][:S]) if summary_only else (Kr[j], V[j])
    outs = []
    for t in range(T):
        q = rot(Q[t], t)
        o, l = gca.stream_step(q[None], t, fkv, n=n, k=k, S=S, scale=0.125, impl="np")
        outs.append(o[0])
    return np.stack(outs)


def test_gca_output_does_not_move_with_a_common_time_shift():
    a = _rope_stream(9, 0)
    b = _rope_stream(9, 1234)
    assert np.abs(a - b).max() < 2e-5
    # and the encoding matters: without it the outputs differ
    c = _rope_stream(9, 0, rope=False)
    assert np.abs(a - c).max() > 1e-2


def test_planted_rotation_of_keys_only_is_caught(monkeypatch):
    # a mistake that rotates K but leaves Q unrotated breaks the shift invariance
    real = gca.rope_frame
    calls = {"n": 0}

    def keys_only(x, frame, **kw):
        calls["n"] += 1
        return real(x, frame, **kw) if calls["n"] <= 9 else x.astype(np.float32)
    monkeypatch.setattr(gca, "rope_frame", keys_only)
    a = _rope_stream(9, 0)
    calls["n"] = 0
    b = _rope_stream(9, 1234)
    assert np.abs(a - b).max() > 1e-3


def test_planted_pairing_of_distant_dims_is_caught(monkeypatch):
    # rotating (d, d+32) pairs instead of (2i, 2i+1) changes what each axis owns
    real = gca.rope_matrix

    def half_split(t, y, x, D=64, base=gca.ROPE_BASE, split=gca.ROPE_SPLIT):
        R = real(t, y, x, D, base, split)
        perm = np.array([d // 2 if d % 2 == 0 else 32 + d // 2 for d in range(D)])
        P = np.eye(D)[perm]
        return P.T @ R @ P
    monkeypatch.setattr(gca, "rope_matrix", half_split)
    with pytest.raises(AssertionError):
        test_each_axis_owns_its_dims()
