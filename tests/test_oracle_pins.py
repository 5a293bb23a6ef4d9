"""Pins of the CPU oracle to facts fixed outside it (CPU only).

Each pin compares the oracle with something it does not contain: numbers the
LingBot-Map pages print (token counts, the n=2/k=2 mask picture), a library
routine (torch SDPA in fp64 on the CPU) in the cases where GCA reduces to plain
or frame-causal attention, closed-form invariants, and a brute-force
formulation of the same rule.  The mutation tests at the end plant plausible
mistakes into the oracle and check that some pin fails.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import gca
from oracle.allocator import PageTableSim, CapacityError, StateError
from windowed_memory_attention_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_stream(T, M, H, D, seed, S=6):
    rng = np.random.default_rng(seed)
    shape = (T, S + M, H, D)
    return (rng.standard_normal(shape).astype(np.float32),
            rng.standard_normal(shape).astype(np.float32),
            rng.standard_normal(shape).astype(np.float32))


def _frame_kv(K, V):
    def get(j, summary_only):
        return K[j], V[j]
    return get


def _o1_all_frames(Q, K, V, *, n, k, S, scale, impl="np"):
    outs, lses = [], []
    for i in range(Q.shape[0]):
        o, l = gca.stream_step(Q[i:i + 1], i, _frame_kv(K, V), n=n, k=k, S=S,
                               scale=scale, impl=impl)
        outs.append(o[0])
        lses.append(l[0])
    return np.stack(outs), np.stack(lses)


def _sdpa_block_causal(Q, K, V, scale):
    """Frame-causal attention through torch's SDPA (fp64, CPU, explicit mask)."""
    T, Lq, H, D = Q.shape
    q = torch.from_numpy(Q.astype(np.float64)).reshape(T * Lq, H, D).permute(1, 0, 2)
    k = torch.from_numpy(K.astype(np.float64)).reshape(T * Lq, H, D).permute(1, 0, 2)
    v = torch.from_numpy(V.astype(np.float64)).reshape(T * Lq, H, D).permute(1, 0, 2)
    fr = torch.arange(T).repeat_interleave(Lq)
    mask = fr[None, :] <= fr[:, None]
    out = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None],
                                                           attn_mask=mask, scale=scale)
    return out[0].permute(1, 0, 2).reshape(T, Lq, H, D).numpy()


# ----------------------------------------------------------------------------
# pins
# ----------------------------------------------------------------------------
def pin_token_counts():
    g = json.load(open(os.path.join(GOLDEN, "token_counts.json")))
    M, S, n, k, T = g["M"], g["S"], g["n"], g["k"], g["T"]
    ok = gca.cache_tokens(M, S, n, k, T) == g["gca_tokens"]
    ok &= gca.cache_tokens(M, S, n, k, 0) + 0 == 0
    ok &= M * (n + k) == g["gca_tokens_fixed_part"]
    ok &= gca.causal_tokens(M, S, T) == g["causal_tokens"]
    ok &= round(gca.causal_tokens(M, S, T) / gca.cache_tokens(M, S, n, k, T)) == g["ratio_rounded"]
    return bool(ok)


def pin_mask_picture():
    lines = [l.strip() for l in open(os.path.join(GOLDEN, "visibility_n2_k2.txt"))
             if l.strip() and not l.startswith("#")]
    T = len(lines)
    got = gca.frame_visibility_matrix(T, n=2, k=2, S=6)
    if got != lines:
        return False
    # the streaming simulator must paint the same picture
    for i in range(T):
        full, summ = gca.stream_state(i, n=2, k=2)
        row = "".join("F" if j in full else ("S" if j in summ else ".") for j in range(T))
        if row != lines[i]:
            return False
    return True


def pin_streamed_key_count(M=5, S=6, n=2, k=3, T=12, H=1, D=8):
    """With Q = 0 every visible key gets the same weight, so lse = ln(#visible)
    — the cache-size closed form — and the output is the mean visible V."""
    Q, K, V = _rand_stream(T, M, H, D, seed=7, S=S)
    Q[:] = 0
    _, lse = _o1_all_frames(Q, K, V, n=n, k=k, S=S, scale=0.125)
    for i in range(T):
        want = math.log(gca.cache_tokens(M, S, n, k, i + 1))
        if not np.allclose(lse[i], want, atol=1e-12, rtol=0):
            return False
    return True


def pin_causal_limit_sdpa(M=7, n=2, k=6, T=6, H=2, D=16, seed=3):
    """T <= n+k: nothing is evicted and GCA is frame-causal attention."""
    Q, K, V = _rand_stream(T, M, H, D, seed)
    scale = 1 / math.sqrt(D)
    ref = _sdpa_block_causal(Q, K, V, scale)
    o1, _ = _o1_all_frames(Q, K, V, n=n, k=k, S=6, scale=scale)
    o2, _ = gca.bruteforce(Q, K, V, n=n, k=k, S=6, scale=scale)
    return bool(np.abs(o1 - ref).max() < 1e-12 and np.abs(o2 - ref).max() < 1e-12)


def _o1_keyframes(Q, K, V, *, n, k, S, interval, scale, impl="np"):
    """O1 over a stream in which only keyframes are cached: keyframes through
    stream_step on the keyframe sequence, the others through transient_step."""
    keys = [y for y in range(Q.shape[0]) if gca.is_keyframe(y, n=n, interval=interval)]
    fkv = _frame_kv(K[keys], V[keys])
    outs, lses = [], []
    for x in range(Q.shape[0]):
        i = gca.latest_keyframe(x, n=n, interval=interval)
        if gca.is_keyframe(x, n=n, interval=interval):
            o, l = gca.stream_step(Q[x:x + 1], i, fkv, n=n, k=k, S=S, scale=scale, impl=impl)
            o, l = o[0], l[0]
        else:
            o, l = gca.transient_step(Q[x], K[x], V[x], i, fkv, n=n, k=k, S=S, scale=scale,
                                      impl=impl)
        outs.append(o)
        lses.append(l)
    return np.stack(outs), np.stack(lses)


def pin_transient_before_eviction_is_sdpa(M=5, n=2, k=8, X=9, interval=2, H=2, D=16, seed=21):
    """While nothing has been evicted a non-keyframe sees every token of the
    cached keyframes and of itself: plain attention (torch SDPA, fp64)."""
    Q, K, V = _rand_stream(X, M, H, D, seed)
    scale = 1 / math.sqrt(D)
    keys = [y for y in range(X) if gca.is_keyframe(y, n=n, interval=interval)]
    assert len(keys) <= n + k                      # no eviction in this stream
    fkv = _frame_kv(K[keys], V[keys])
    checked = 0
    for x in range(X):
        if gca.is_keyframe(x, n=n, interval=interval):
            continue
        i = gca.latest_keyframe(x, n=n, interval=interval)
        o, _ = gca.transient_step(Q[x], K[x], V[x], i, fkv, n=n, k=k, S=6, scale=scale, impl="np")
        seen = keys[:i + 1] + [x]
        kk = torch.from_numpy(K[seen].astype(np.float64)).reshape(-1, H, D).permute(1, 0, 2)
        vv = torch.from_numpy(V[seen].astype(np.float64)).reshape(-1, H, D).permute(1, 0, 2)
        qq = torch.from_numpy(Q[x].astype(np.float64)).permute(1, 0, 2)
        ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, scale=scale)
        if np.abs(o - ref.permute(1, 0, 2).numpy()).max() > 1e-12:
            return False
        checked += 1
    return checked > 0


def pin_transient_key_count(M=5, S=6, n=2, k=3, X=17, interval=3, H=1, D=8):
    """Q = 0: lse = ln(#keys read) = ln(cache size after the latest keyframe
    (closed form) + the frame's own S+M tokens)."""
    Q, K, V = _rand_stream(X, M, H, D, seed=9, S=S)
    Q[:] = 0
    try:
        _, lse = _o1_keyframes(Q, K, V, n=n, k=k, S=S, interval=interval, scale=0.125)
    except (ValueError, IndexError):
        return False                  # an oracle that cannot even run fails the pin
    for x in range(X):
        # keyframes among video frames 0..x, counted directly: all of the first
        # n, then frames n, n+interval, n+2*interval, ...
        cached = x + 1 if x < n else n + (x - n) // interval + 1
        own = 0 if (x < n or (x - n) % interval == 0) else S + M
        want = math.log(gca.cache_tokens(M, S, n, k, cached) + own)
        if not np.allclose(lse[x], want, atol=1e-12, rtol=0):
            return False
    return True


def pin_sliding_window_is_banded_sdpa(M=5, k=3, T=9, H=2, D=16, seed=17):
    """No anchors and no trajectory memory (keep = 0): frame i sees every token
    of frames i-k+1..i and nothing else — the sliding-window mask of the mask
    figure (c), here an explicit frame band through torch SDPA (fp64)."""
    Q, K, V = _rand_stream(T, M, H, D, seed)
    scale = 1 / math.sqrt(D)
    Lq = M + 6
    q = torch.from_numpy(Q.astype(np.float64)).reshape(T * Lq, H, D).permute(1, 0, 2)
    kk = torch.from_numpy(K.astype(np.float64)).reshape(T * Lq, H, D).permute(1, 0, 2)
    vv = torch.from_numpy(V.astype(np.float64)).reshape(T * Lq, H, D).permute(1, 0, 2)
    fr = torch.arange(T).repeat_interleave(Lq)
    band = (fr[None, :] <= fr[:, None]) & (fr[None, :] >= fr[:, None] - k + 1)
    ref = torch.nn.functional.scaled_dot_product_attention(q[None], kk[None], vv[None], attn_mask=band,
                                                           scale=scale)
    ref = ref[0].permute(1, 0, 2).reshape(T, Lq, H, D).numpy()
    o1 = []
    for i in range(T):
        o, _ = gca.stream_step(Q[i:i + 1], i, _frame_kv(K, V), n=0, k=k, S=6, scale=scale,
                               impl="np", keep=0)
        o1.append(o[0])
    o2, _ = gca.bruteforce(Q, K, V, n=0, k=k, S=6, scale=scale, keep=0)
    return bool(np.abs(np.stack(o1) - ref).max() < 1e-12 and np.abs(o2 - ref).max() < 1e-12)


def pin_camera_only_key_count(M=5, S=6, n=2, k=3, T=12, H=1, D=8):
    """Camera-only memory (keep = 1), Q = 0: lse = ln(#keys), and #keys is every
    token of the min(T, n+k) full frames plus one camera token per other frame."""
    Q, K, V = _rand_stream(T, M, H, D, seed=29, S=S)
    Q[:] = 0
    for i in range(T):
        _, lse = gca.stream_step(Q[i:i + 1], i, _frame_kv(K, V), n=n, k=k, S=S, scale=0.125,
                                 impl="np", keep=1)
        full = min(i + 1, n + k)
        want = math.log((M + S) * full + (i + 1 - full))
        if not np.allclose(lse[0], want, atol=1e-12, rtol=0):
            return False
    return True


# ----------------------------------------------------------------------------
# tests
# ----------------------------------------------------------------------------
def test_token_counts_match_worked_example():
    assert pin_token_counts()


def test_allocator_resident_tokens_follow_closed_form():
    # the pages' worked example streamed to T=10000 with eviction after each append
    sim = PageTableSim(M=500, S=6, P=128, n=3, k=16, max_frames=10000)
    for T in range(1, 10001):
        sim.append()
        sim.evict()
        assert sim.resident_tokens() == gca.cache_tokens(500, 6, 3, 16, T)
    assert sim.resident_tokens() == 69500
    # tokens reachable through the walk list equal the closed form too
    assert sum(e[4] for e in sim.walk()) == 69500


def test_mask_picture_n2_k2():
    assert pin_mask_picture()


def test_lse_of_zero_query_counts_the_cache():
    assert pin_streamed_key_count()


def test_causal_limit_equals_sdpa():
    assert pin_causal_limit_sdpa()
    # the dense-cache workload's regime: k >= T, several frames
    assert pin_causal_limit_sdpa(M=9, n=3, k=40, T=5, H=3, D=8, seed=11)


def test_transient_before_eviction_equals_sdpa():
    assert pin_transient_before_eviction_is_sdpa()
    assert pin_transient_before_eviction_is_sdpa(M=9, n=1, k=6, X=11, interval=3, seed=4)


def test_transient_lse_counts_cache_and_own_tokens():
    assert pin_transient_key_count()
    assert pin_transient_key_count(n=3, k=2, X=14, interval=2)


def test_keyframe_schedule_follows_the_walkthrough():
    # scale frames always enter; then every interval-th frame counted from n
    assert [gca.is_keyframe(x, n=3, interval=2) for x in range(9)] == \
        [True, True, True, True, False, True, False, True, False]
    assert all(gca.is_keyframe(x, n=3, interval=1) for x in range(20))
    assert [gca.latest_keyframe(x, n=3, interval=2) for x in range(9)] == [0, 1, 2, 3, 3, 4, 4, 5, 5]


@pytest.mark.parametrize("interval,anchor_block", [(2, False), (3, False), (2, True)])
def test_keyframe_stream_equals_bruteforce(interval, anchor_block):
    M, n, k, X, H, D = 4, 2, 3, 16, 2, 8
    Q, K, V = _rand_stream(X, M, H, D, seed=13 + interval)
    scale = 1 / math.sqrt(D)
    keys = [y for y in range(X) if gca.is_keyframe(y, n=n, interval=interval)]
    fkv = _frame_kv(K[keys], V[keys])
    o2, l2 = gca.bruteforce_keyframes(Q, K, V, n=n, k=k, S=6, interval=interval, scale=scale,
                                      anchor_block=anchor_block)
    for x in range(X):
        i = gca.latest_keyframe(x, n=n, interval=interval)
        if gca.is_keyframe(x, n=n, interval=interval):
            if anchor_block and i < n:
                continue                     # the anchor block is one query block, not streamed
            o, l = gca.stream_step(Q[x:x + 1], i, fkv, n=n, k=k, S=6, scale=scale,
                                   anchor_block=anchor_block, impl="np")
            o, l = o[0], l[0]
        else:
            o, l = gca.transient_step(Q[x], K[x], V[x], i, fkv, n=n, k=k, S=6, scale=scale,
                                      anchor_block=anchor_block, impl="np")
        assert np.abs(o - o2[x]).max() < 1e-12
        assert np.abs(l - l2[x]).max() < 1e-12


def test_transient_with_constant_values():
    Q, K, V = _rand_stream(7, 5, 2, 8, seed=3)
    V[:] = 2.5
    keys = [0, 1, 2, 4, 6]
    o, _ = gca.transient_step(Q[5], K[5], V[5], 3, _frame_kv(K[keys], V[keys]), n=2, k=2, S=6,
                              scale=0.3, impl="np")
    assert np.abs(o - 2.5).max() < 1e-12


def test_sliding_window_mask_equals_banded_sdpa():
    assert pin_sliding_window_is_banded_sdpa()
    assert pin_sliding_window_is_banded_sdpa(M=3, k=1, T=5, seed=2)


def test_camera_only_key_count():
    assert pin_camera_only_key_count()
    assert pin_camera_only_key_count(n=0, k=2, T=9)
    # the closed form agrees with the per-step count
    for T in (1, 5, 40):
        assert gca.cache_tokens(500, 6, 3, 16, T, keep=1) == 505 * min(T, 19) + T
        assert gca.cache_tokens(500, 6, 0, 16, T, keep=0) == 506 * min(T, 16)


@pytest.mark.parametrize("keep,n,anchor_block", [(1, 2, False), (0, 2, False), (1, 2, True), (0, 0, False)])
def test_memory_variants_stream_equals_bruteforce(keep, n, anchor_block):
    M, k, T, H, D = 4, 3, 10, 2, 8
    Q, K, V = _rand_stream(T, M, H, D, seed=31 + keep)
    scale = 1 / math.sqrt(D)
    o2, l2 = gca.bruteforce(Q, K, V, n=n, k=k, S=6, scale=scale, anchor_block=anchor_block, keep=keep)
    for i in range(T):
        if anchor_block and i < n:
            continue
        o, l = gca.stream_step(Q[i:i + 1], i, _frame_kv(K, V), n=n, k=k, S=6, scale=scale,
                               anchor_block=anchor_block, impl="np", keep=keep)
        assert np.abs(o[0] - o2[i]).max() < 1e-12
        assert np.abs(l[0] - l2[i]).max() < 1e-12


@pytest.mark.parametrize("keep", [6, 1, 0])
def test_allocator_memory_variants_follow_closed_form(keep):
    n = 0 if keep == 0 else 3
    sim = PageTableSim(M=500, S=6, P=128, n=n, k=16, max_frames=400, keep=keep)
    for T in range(1, 401):
        sim.append()
        sim.evict()
        want = gca.cache_tokens(500, 6, n, 16, T, keep=keep)
        assert sim.resident_tokens() == want
        assert sum(e[4] for e in sim.walk()) == want
    assert sim.ipf == math.ceil((500 + 6 - keep) / 128)
    # token slots: kept tokens in the stream, the others in the frame's image pages in order
    t = 399
    for tau in range(506):
        pid, slot = sim.slot_of(t, tau)
        if tau < keep:
            assert pid in sim.summary_pages and slot == (keep * t + tau) % 128
        else:
            assert pid == sim.image_pages[t][(tau - keep) // 128] and slot == (tau - keep) % 128


@pytest.mark.parametrize("keep,n", [(1, 2), (0, 0)])
def test_transient_key_count_with_memory_variants(keep, n):
    """A non-keyframe over a camera-only or memory-free cache: Q = 0 gives
    lse = ln(every token of the min(K, n+k) full keyframes + keep tokens of the
    other K keyframes + the frame's own S+M), K = keyframes cached so far."""
    M, S, k, X, interval = 5, 6, 3, 15, 2
    Q, K, V = _rand_stream(X, M, 1, 8, seed=41, S=S)
    Q[:] = 0
    keys = [y for y in range(X) if gca.is_keyframe(y, n=n, interval=interval)]
    fkv = _frame_kv(K[keys], V[keys])
    for x in range(X):
        if gca.is_keyframe(x, n=n, interval=interval):
            continue
        cached = x + 1 if x < n else n + (x - n) // interval + 1
        _, lse = gca.transient_step(Q[x], K[x], V[x], cached - 1, fkv, n=n, k=k, S=S,
                                    scale=0.125, impl="np", keep=keep)
        full = min(cached, n + k)
        want = math.log((M + S) * full + keep * (cached - full) + (M + S))
        assert np.allclose(lse, want, atol=1e-12, rtol=0), x


def test_single_frame_is_plain_attention():
    Q, K, V = _rand_stream(1, 11, 2, 16, seed=5)
    scale = 0.25
    o, lse = gca.stream_step(Q, 0, _frame_kv(K, V), n=3, k=4, S=6, scale=scale, impl="np")
    q = torch.from_numpy(Q[0].astype(np.float64)).permute(1, 0, 2)
    k = torch.from_numpy(K[0].astype(np.float64)).permute(1, 0, 2)
    v = torch.from_numpy(V[0].astype(np.float64)).permute(1, 0, 2)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=scale)
    assert np.abs(o[0] - ref.permute(1, 0, 2).numpy()).max() < 1e-12
    s = torch.einsum("hrd,hud->hru", q, k) * scale
    assert np.abs(lse[0] - torch.logsumexp(s, -1).T.numpy()).max() < 1e-12


@pytest.mark.parametrize("M,n,k,T,H,D,seed", [
    (16, 3, 4, 32, 2, 64, 0),      # the tiny workload's shape
    (5, 1, 1, 9, 1, 8, 1),         # window of one frame (only the current frame)
    (3, 0, 2, 8, 2, 4, 2),         # no anchors
    (7, 2, 3, 10, 3, 8, 3),
])
def test_streaming_equals_bruteforce(M, n, k, T, H, D, seed):
    Q, K, V = _rand_stream(T, M, H, D, seed)
    scale = 1 / math.sqrt(D)
    o1, l1 = _o1_all_frames(Q, K, V, n=n, k=k, S=6, scale=scale, impl="c")
    o2, l2 = gca.bruteforce(Q, K, V, n=n, k=k, S=6, scale=scale)
    assert np.abs(o1 - o2).max() < 1e-12
    assert np.abs(l1 - l2).max() < 1e-12


def test_tiny_workload_from_generator_streaming_equals_bruteforce():
    w = inputs.TINY
    Q = np.stack([inputs.draw(w, t, "q")[0].numpy() for t in range(w.T)])
    K = np.stack([inputs.draw(w, t, "k")[0].numpy() for t in range(w.T)])
    V = np.stack([inputs.draw(w, t, "v")[0].numpy() for t in range(w.T)])
    o1, _ = _o1_all_frames(Q, K, V, n=w.n, k=w.k, S=w.S, scale=w.softmax_scale, impl="c")
    o2, _ = gca.bruteforce(Q, K, V, n=w.n, k=w.k, S=w.S, scale=w.softmax_scale)
    assert np.abs(o1 - o2).max() < 1e-12


@pytest.mark.parametrize("F,last", [(2, 9), (4, 11), (3, 7)])
def test_multi_frame_block_equals_bruteforce(F, last):
    M, n, k, H, D = 6, 2, 4, 2, 8
    T = last + 1
    Q, K, V = _rand_stream(T, M, H, D, seed=F)
    scale = 0.3
    o, l = gca.stream_step(Q[last - F + 1:last + 1], last, _frame_kv(K, V), n=n, k=k,
                           S=6, scale=scale, impl="np")
    o2, l2 = gca.bruteforce(Q, K, V, n=n, k=k, S=6, scale=scale)
    assert np.abs(o - o2[last - F + 1:last + 1]).max() < 1e-12


def test_anchor_block_equals_bruteforce():
    M, n, k, H, D, T = 5, 3, 2, 2, 8, 9
    Q, K, V = _rand_stream(T, M, H, D, seed=4)
    o2, _ = gca.bruteforce(Q, K, V, n=n, k=k, S=6, scale=0.3, anchor_block=True)
    o, _ = gca.stream_step(Q[:n], n - 1, _frame_kv(K, V), n=n, k=k, S=6, scale=0.3,
                           anchor_block=True, impl="np")
    assert np.abs(o - o2[:n]).max() < 1e-12
    for i in range(n, T):
        o, _ = gca.stream_step(Q[i:i + 1], i, _frame_kv(K, V), n=n, k=k, S=6, scale=0.3,
                               anchor_block=True, impl="np")
        assert np.abs(o[0] - o2[i]).max() < 1e-12
    # the anchors see each other in full: frame 0 attends to frame 2's image tokens
    assert gca.visible(0, 2, 6, n=n, k=k, S=6, anchor_block=True)
    assert not gca.visible(0, 2, 6, n=n, k=k, S=6, anchor_block=False)


def test_constant_values_give_constant_output():
    Q, K, V = _rand_stream(12, 6, 2, 8, seed=9)
    V[:] = 0.375
    o, _ = _o1_all_frames(Q, K, V, n=2, k=3, S=6, scale=0.3, impl="c")
    assert np.abs(o - 0.375).max() < 1e-12


def test_key_order_does_not_matter():
    rng = np.random.default_rng(1)
    q = rng.standard_normal((5, 2, 8)).astype(np.float32)
    k = rng.standard_normal((40, 2, 8)).astype(np.float32)
    v = rng.standard_normal((40, 2, 8)).astype(np.float32)
    perm = rng.permutation(40)
    a, la = gca.attention_c(q, k, v, 0.3)
    b, lb = gca.attention_c(q, k[perm], v[perm], 0.3)
    assert np.abs(a - b).max() < 1e-12 and np.abs(la - lb).max() < 1e-12


def test_c_core_matches_numpy_twin():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((9, 3, 64)).astype(np.float32)
    k = (rng.standard_normal((300, 3, 64)) * 3).astype(np.float32)
    v = rng.standard_normal((300, 3, 64)).astype(np.float32)
    a, la = gca.attention_c(q, k, v, 0.125)
    b, lb = gca.attention_np(q, k, v, 0.125)
    assert np.abs(a - b).max() < 1e-12 and np.abs(la - lb).max() < 1e-11


# ----------------------------------------------------------------------------
# page-table simulator
# ----------------------------------------------------------------------------
def test_allocator_smallest_free_first_and_layout():
    sim = PageTableSim(M=16, S=6, P=128, n=3, k=4, max_frames=32)
    # capacity: (3+4+1) frames x 1 image page + ceil(6*32/128) = 2 summary pages
    assert sim.num_pages == 10
    t = sim.append()
    assert t == 0 and sim.summary_pages == [0] and sim.image_pages[0] == [1]
    for _ in range(7):
        sim.append()
        sim.evict()
    # frames 0..7: pages 1..8 in order; nothing evicted before frame 7 (k=4, n=3)
    assert [sim.image_pages[f][0] for f in sorted(sim.image_pages)] == [1, 2, 3, 5, 6, 7, 8]
    # frame 3 left the window after frame 7 and gave back page 4
    assert list(sim.free) == [4, 9]
    sim.append()                  # frame 8 takes the smallest free page
    assert sim.image_pages[8] == [4]


def test_allocator_summary_stream_crosses_pages():
    sim = PageTableSim(M=3, S=6, P=64, n=1, k=1, max_frames=40)
    seen = {}
    for t in range(40):
        sim.append()
        sim.evict()
        for s in range(6):
            pid, slot = sim.slot_of(t, s)
            assert (6 * t + s) % 64 == slot
            assert (pid, slot) not in seen
            seen[(pid, slot)] = (t, s)
    assert len(sim.summary_pages) == math.ceil(240 / 64)
    w = sim.walk()
    summ = [e for e in w if e[1] == 1]
    assert [e[3] for e in summ] == [0, 64, 128, 192]
    assert [e[4] for e in summ] == [64, 64, 64, 48]
    assert [e[2] for e in summ] == [0, 10, 21, 32]


def test_allocator_capacity_and_state_errors():
    sim = PageTableSim(M=16, S=6, P=128, n=3, k=4, max_frames=3)
    for _ in range(3):
        sim.append()
    with pytest.raises(CapacityError):
        sim.append()
    sim2 = PageTableSim(M=16, S=6, P=128, n=1, k=2, max_frames=20)
    for _ in range(6):
        sim2.append()
        sim2.evict()
    with pytest.raises(StateError):
        sim2.walk(F=2)        # frame 3 (window of query frame 4) was evicted
    assert len(sim2.walk(F=1)) > 0
    sim3 = PageTableSim(M=16, S=6, P=128, n=1, k=2, max_frames=20, max_query_frames=3)
    for _ in range(3):
        sim3.append()
    sim3.evict()
    for _ in range(3):
        sim3.append()        # a block of 3 frames appended before any eviction
    assert len(sim3.walk(F=3)) > 0
    with pytest.raises(CapacityError):
        sim3.append()


def test_allocator_reset_matches_fresh_windowed_stream():
    """The windowed workload: reset at every window start gives the same page
    tables as a fresh cache, for all 179 windows of the 20000-frame stream."""
    w = inputs.WINDOWED_VO
    wins = w.windows()
    assert len(wins) == 179 and wins[-1] == (19936, 64)
    assert sum(l for _, l in wins) == 20000 + 16 * 178
    sim = PageTableSim(M=w.M, S=w.S, P=128, n=w.n, k=w.k, max_frames=w.window_frames)
    fresh_walks = []
    ref = PageTableSim(M=w.M, S=w.S, P=128, n=w.n, k=w.k, max_frames=w.window_frames)
    for t in range(w.window_frames):
        ref.append()
        ref.evict()
        fresh_walks.append(ref.walk())
    for start, ln in wins:
        sim.reset()
        for t in range(ln):
            sim.append()
            sim.evict()
            assert sim.walk() == fresh_walks[t]


# ----------------------------------------------------------------------------
# planted mistakes: each must make some pin fail
# ----------------------------------------------------------------------------
def test_planted_window_off_by_one_is_caught(monkeypatch):
    orig = gca.visible

    def wrong(i, j, tau, *, n, k, S, anchor_block=False, keep=None):
        if tau >= S and j <= i and j >= n:
            return j >= i - k             # window one frame too wide
        return orig(i, j, tau, n=n, k=k, S=S, anchor_block=anchor_block, keep=keep)
    monkeypatch.setattr(gca, "visible", wrong)
    assert not pin_mask_picture()


def test_planted_eviction_off_by_one_is_caught(monkeypatch):
    orig = gca.stream_state

    def wrong(i, *, n, k, anchor_block=False):
        return orig(i, n=n, k=k + 1, anchor_block=anchor_block)
    monkeypatch.setattr(gca, "stream_state", wrong)
    assert not pin_mask_picture()
    assert not pin_streamed_key_count()


def test_planted_dropped_summary_tokens_are_caught(monkeypatch):
    orig = gca.stream_state

    def wrong(i, *, n, k, anchor_block=False):
        full, _ = orig(i, n=n, k=k, anchor_block=anchor_block)
        return full, []
    monkeypatch.setattr(gca, "stream_state", wrong)
    assert not pin_streamed_key_count()


def test_planted_wrong_scale_is_caught(monkeypatch):
    orig = gca.attention_np
    monkeypatch.setattr(gca, "attention_np", lambda q, k, v, scale: orig(q, k, v, 1.0))
    assert not pin_causal_limit_sdpa()


def test_planted_swapped_operands_are_caught(monkeypatch):
    orig = gca.attention_np
    monkeypatch.setattr(gca, "attention_np", lambda q, k, v, scale: orig(q, v, k, scale))
    assert not pin_causal_limit_sdpa()


def test_planted_future_frame_leak_is_caught(monkeypatch):
    orig = gca.visible

    def wrong(i, j, tau, *, n, k, S, anchor_block=False, keep=None):
        if j == i + 1 and tau < S:
            return True
        return orig(i, j, tau, n=n, k=k, S=S, anchor_block=anchor_block, keep=keep)
    monkeypatch.setattr(gca, "visible", wrong)
    assert not pin_mask_picture()
    assert not pin_causal_limit_sdpa()


def test_planted_transient_without_own_tokens_is_caught(monkeypatch):
    orig = gca.transient_step

    def wrong(q, own_k, own_v, last_key, frame_kv, **kw):
        return orig(q, own_k[:0], own_v[:0], last_key, frame_kv, **kw)
    monkeypatch.setattr(gca, "transient_step", wrong)
    assert not pin_transient_key_count()


def test_planted_transient_reading_one_keyframe_late_is_caught(monkeypatch):
    orig = gca.latest_keyframe

    def wrong(x, *, n, interval):
        return orig(x, n=n, interval=interval) - 1
    monkeypatch.setattr(gca, "latest_keyframe", wrong)
    assert not pin_transient_key_count()


def test_planted_camera_only_keeping_every_summary_token_is_caught(monkeypatch):
    orig = gca.gather_keys

    def wrong(i, frame_kv, *, n, k, S, anchor_block=False, keep=None):
        return orig(i, frame_kv, n=n, k=k, S=S, anchor_block=anchor_block, keep=None)
    monkeypatch.setattr(gca, "gather_keys", wrong)
    assert not pin_camera_only_key_count()


def test_planted_sliding_window_with_anchor_leak_is_caught(monkeypatch):
    orig = gca.visible

    def wrong(i, j, tau, *, n, k, S, anchor_block=False, keep=None):
        if j == 0 and j <= i:
            return True                   # frame 0 treated as an anchor
        return orig(i, j, tau, n=n, k=k, S=S, anchor_block=anchor_block, keep=keep)
    monkeypatch.setattr(gca, "visible", wrong)
    assert not pin_sliding_window_is_banded_sdpa()


def test_planted_camera_only_keeping_the_wrong_token_is_caught(monkeypatch):
    # keeps one token per old frame, but the anchor token (slot 1) instead of the
    # camera token (slot 0): the key count is unchanged, the brute force differs
    orig = gca.gather_keys

    def wrong(i, frame_kv, *, n, k, S, anchor_block=False, keep=None):
        if keep != 1:
            return orig(i, frame_kv, n=n, k=k, S=S, anchor_block=anchor_block, keep=keep)
        shifted = lambda j, summary_only: tuple(a[1:] for a in frame_kv(j, summary_only))
        full, summary = gca.stream_state(i, n=n, k=k, anchor_block=anchor_block)
        ks, vs = [], []
        for f in full:
            kf, vf = frame_kv(f, False)
            ks.append(kf)
            vs.append(vf)
        for f in summary:
            kf, vf = shifted(f, True)
            ks.append(kf[:1])
            vs.append(vf[:1])
        return np.concatenate(ks, 0), np.concatenate(vs, 0)
    monkeypatch.setattr(gca, "gather_keys", wrong)
    with pytest.raises(AssertionError):
        test_memory_variants_stream_equals_bruteforce(1, 2, False)
