"""GPU parity on inputs built to reach the bf16 kernel's rarer softmax paths.

* The exact-softmax branch partway through a head: the kernel exponentiates
  each page against the row's running max and keeps that result while the
  page's sum stays below 2^64.  A page whose scores rise more than ~64 in
  log2 units above the running max fails that test: the kernel then takes
  the page max, rescales the output accumulated so far by 2^(m_old - m_new)
  and redoes the page's exponentials.  The inputs below place one key whose
  score is 60 nats (86.6 in log2 units) above anything seen before in a page
  that comes after the head's first page, for a third of the rows, and a
  second, larger one in a later page for some of them; the other rows stay on
  the fast path.  Without the rescale those rows' earlier output would keep a
  weight 2^80 too large.
* Masked key slots: slots past a page's stored tokens carry stale bytes.  The
  tests fill them with the largest finite bf16 value in K and V; a masked key
  must get weight exactly 0 (its score is -inf before the exponential), so the
  output still matches the oracle.
* Attending before or after gca_evict_to_summary gives identical bytes: the
  walk list holds only the frames the query block may see.
"""
import numpy as np
import pytest
import torch

from oracle.allocator import PageTableSim
from windowed_memory_attention_b200 import gca, inputs
from gca_stream_util import Mirror, attend, max_err, oracle_step, pool_view

pytestmark = pytest.mark.gpu

TOL = 2e-2
BF16_MAX = 3.3895313892515355e38


def _big_key_stream(w, T, big):
    """Stream T frames; `big` maps frame -> list of (token slot, value on dim 0)
    of keys made large along head dim 0 (all other dims zero)."""
    cache = gca.Cache.for_workload(w)
    mirror = Mirror(w, [0])
    for t in range(T):
        k = inputs.draw(w, t, "k", "cuda")
        v = inputs.draw(w, t, "v", "cuda")
        for tau, gamma in big.get(t, []):
            k[:, tau] = 0
            k[:, tau, :, 0] = gamma
        cache.append(k, v)
        cache.evict()
        mirror.record(t, k, v, keep_full=True)
    return cache, mirror


def _query(w, t, lift):
    """Frame t's queries with dim 0 set to `lift` on rows r % 3 == 0 and to 0
    elsewhere, so only those rows see the large keys."""
    q = inputs.draw(w, t, "q", "cuda")
    rows = torch.arange(w.Lq, device="cuda")
    sel = (rows % 3 == 0)
    q[:, :, :, 0] = 0
    q[:, sel, :, 0] = lift
    return q, sel


@pytest.mark.parametrize("case", ["tiny", "worked_shape"])
def test_exact_branch_mid_head_rescales_the_output(case):
    if case == "tiny":
        # tiny bf16: one 128-slot image page per frame, walk = anchors 0..2,
        # window frames, then the summary pages
        w, T = inputs.TINY_BF16.with_(T=12), 12
        late = T - 1
        big = {late: [(w.S + 3, 120.0)],             # image token of the current frame
               T - 3: [(0, 160.0)]}                  # summary token of an older window frame
    else:
        # the worked example's shape (4 image pages per frame, 16 heads) on a
        # short stream: the large keys sit in the last image pages
        w, T = inputs.WORKED_EXAMPLE.with_(T=24, key_norm_sigma=None), 24
        late = T - 1
        big = {late: [(w.S + 400, 120.0)], T - 2: [(w.S + 130, 140.0)]}
    cache, mirror = _big_key_stream(w, T, big)
    q, sel = _query(w, late, 4.0)
    # the margin: lifted rows score 4 * 120 / 8 = 60 nats = 86.6 log2 units on
    # the first large key, far above the 2^64 page-sum threshold
    assert 4.0 * 120.0 * w.softmax_scale / np.log(2.0) > 64 + 20
    out, lse = attend(cache, 0, q)
    want, wlse = oracle_step(mirror, 0, q.float().cpu().numpy(), late)
    torch.cuda.synchronize()
    assert max_err(out, want) <= TOL
    assert max_err(lse, wlse) <= TOL
    # the lifted rows are dominated by the large keys' values; the others are not
    got = out[0].float().cpu().numpy()
    assert np.isfinite(got).all()
    assert cache.status() == 0
    # control: the same stream and rows with the lift removed stay on the fast path
    q0 = q.clone()
    q0[:, :, :, 0] = 0
    out0, _ = attend(cache, 0, q0)
    want0, _ = oracle_step(mirror, 0, q0.float().cpu().numpy(), late)
    torch.cuda.synchronize()
    assert max_err(out0, want0) <= TOL
    assert float((out[0, sel.cpu()] - out0[0, sel.cpu()]).abs().max()) > 0.5


@pytest.mark.parametrize("page_size", [128, 64])
def test_masked_slots_get_exactly_zero_weight(page_size):
    # tiny bf16, 16 image tokens per frame: slots 16.. of every image page and
    # the tail of the last summary page are masked
    w = inputs.TINY_BF16.with_(T=14, page_size=page_size)
    cache = gca.Cache.for_workload(w)
    mirror = Mirror(w, [0])
    for t in range(w.T):
        k, v = inputs.draw(w, t, "k", "cuda"), inputs.draw(w, t, "v", "cuda")
        cache.append(k, v)
        cache.evict()
        mirror.record(t, k, v, keep_full=True)
    info = cache.info()
    shape = (w.L, info.num_pages, w.H, w.page_size, w.D)
    kp = pool_view(cache, "k", torch.bfloat16).view(shape)
    vp = pool_view(cache, "v", torch.bfloat16).view(shape)
    torch.cuda.synchronize()
    filled = 0
    for pid, kind, frame, first, n_valid in cache.layout():
        if n_valid < w.page_size:
            kp[0, pid, :, n_valid:] = BF16_MAX
            vp[0, pid, :, n_valid:] = BF16_MAX
            filled += w.page_size - n_valid
    assert filled > 0
    q = inputs.draw(w, w.T - 1, "q", "cuda")
    out, lse = attend(cache, 0, q)
    want, wlse = oracle_step(mirror, 0, q.float().cpu().numpy(), w.T - 1)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
    assert max_err(out, want) <= TOL
    assert max_err(lse, wlse) <= TOL
    assert cache.status() == 0


def test_attend_before_or_after_evict_is_identical():
    # gca_attend with an eviction still pending reads the same walk list as
    # after it, so the output bytes are the same
    w = inputs.TINY_BF16.with_(T=16)
    cache = gca.Cache.for_workload(w)
    sim = PageTableSim(M=w.M, S=w.S, P=w.page_size, n=w.n, k=w.k, max_frames=w.T)
    for t in range(w.T):
        k, v = inputs.draw(w, t, "k", "cuda"), inputs.draw(w, t, "v", "cuda")
        cache.append(k, v)
        sim.append()
        q = inputs.draw(w, t, "q", "cuda")
        before = cache.layout()
        out1, lse1 = attend(cache, 0, q)
        evicted = cache.evict()
        assert evicted == sim.evict() == (1 if t >= w.n + w.k else 0)
        assert cache.layout() == before == sim.walk()
        out2, lse2 = attend(cache, 0, q)
        torch.cuda.synchronize()
        assert torch.equal(out1, out2) and torch.equal(lse1, lse2), t
    assert cache.status() == 0


def test_block_attend_comes_before_the_eviction():
    # a block of F=2 frames needs the frame the eviction after its last frame
    # removes: attending first works, attending after it is a state error
    w = inputs.TINY_BF16.with_(T=16)
    F = 2
    cache = gca.Cache.for_workload(w, max_query_frames=F)
    mirror = Mirror(w, [0])
    for t in range(w.T):
        k, v = inputs.draw(w, t, "k", "cuda"), inputs.draw(w, t, "v", "cuda")
        cache.append(k, v)
        mirror.record(t, k, v, keep_full=True)
        if t + 1 >= F:
            q = torch.stack([inputs.draw(w, x, "q", "cuda")[0] for x in range(t + 1 - F, t + 1)])
            out, _ = attend(cache, 0, q, F)
            want, _ = oracle_step(mirror, 0, q.float().cpu().numpy(), t, F=F)
            torch.cuda.synchronize()
            assert max_err(out, want) <= TOL, t
        n_ev = cache.evict()
        if n_ev and t + 1 >= F:
            with pytest.raises(gca.GCAError) as e:
                attend(cache, 0, q, F)
            assert e.value.name == "GCA_ERR_STATE"
    assert cache.status() == 0
