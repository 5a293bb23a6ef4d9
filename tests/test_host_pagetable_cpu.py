"""The library's own page table against the simulator, on the CPU.

A cache created with device = GCA_HOST_ONLY runs the C++ page-table code of
libgca.so (allocation, summary stream, eviction, reset, walk list, token
slots) with no device state, so these comparisons need no GPU.  They are
bit-exact: the walk lists, evicted counts, resident tokens and token slots of
the library equal oracle/allocator.py's at every compared step.
"""
import pytest

from oracle.allocator import PageTableSim, StateError
from windowed_memory_attention_b200 import gca, inputs


def _pair(w, keep=None, **cfg):
    max_frames = cfg.pop("max_frames", w.window_frames or w.T)
    mode = {None: gca.GCA_MEMORY_SUMMARY, 1: gca.GCA_MEMORY_CAMERA, 0: gca.GCA_MEMORY_NONE}[keep]
    cache = gca.Cache.for_workload(w, max_frames=max_frames, device=gca.GCA_HOST_ONLY,
                                   trajectory_memory=mode, **cfg)
    sim = PageTableSim(M=w.M, S=w.S, P=w.page_size, n=w.n, k=w.k, max_frames=max_frames,
                       max_query_frames=cfg.get("max_query_frames", 1),
                       frame_slack=cfg.get("frame_slack", 0),
                       anchor_block=cfg.get("anchor_block", False), keep=keep)
    return cache, sim


def _step(cache, sim):
    t = cache.append(None, None)
    assert t == sim.append()
    assert cache.evict() == sim.evict()
    return t


@pytest.mark.parametrize("w,steps,every", [
    (inputs.WORKED_EXAMPLE, 10000, 97),
    (inputs.METRIC_518x378.with_(L=1), 600, 1),
    (inputs.METRIC_518x378.with_(L=1, page_size=64), 400, 1),
])
def test_stream_tables_match_the_simulator(w, steps, every):
    cache, sim = _pair(w)
    for _ in range(steps):
        t = _step(cache, sim)
        info = cache.info()
        assert info.frames == sim.T and info.resident_tokens == sim.resident_tokens()
        assert info.full_frames == len(sim.image_pages)
        if t < 300 or t % every == 0 or t == steps - 1:
            assert cache.layout() == sim.walk()
    if w is inputs.WORKED_EXAMPLE:
        assert cache.info().resident_tokens == 69500          # the pages' worked example
    cache.close()


@pytest.mark.parametrize("keep,n", [(1, 3), (0, 0), (0, 3)])
def test_memory_variant_tables_match_the_simulator(keep, n):
    w = inputs.WORKED_EXAMPLE.with_(n=n)
    cache, sim = _pair(w, keep=keep, max_frames=700)
    for _ in range(700):
        t = _step(cache, sim)
        assert cache.layout() == sim.walk(), t
        assert cache.info().resident_tokens == sim.resident_tokens()
    cache.close()


def test_token_slots_match_the_simulator():
    for keep in (None, 1, 0):
        w = inputs.TINY.with_(n=3 if keep != 0 else 0)
        cache, sim = _pair(w, keep=keep)
        for _ in range(w.T):
            _step(cache, sim)
        for frame in range(w.T):
            for tau in range(w.Lq):
                try:
                    want = sim.slot_of(frame, tau)
                except KeyError:
                    with pytest.raises(gca.GCAError) as e:
                        cache.token_slot(frame, tau)
                    assert e.value.name == "GCA_ERR_STATE"          # left with the image pages
                    continue
                assert cache.token_slot(frame, tau) == want
        cache.close()


def test_anchor_block_and_multi_frame_walks():
    w = inputs.TINY.with_(T=14)
    F = w.n
    cache, sim = _pair(w, anchor_block=True, max_query_frames=F)
    for t in range(w.T):
        assert cache.append(None, None) == sim.append() == t
        if t == F - 1:                       # the anchor block, before any eviction
            assert cache.layout(F) == sim.walk(F)
        for f in (1, 2):
            if f <= sim.T:
                try:
                    want = sim.walk(f)
                except StateError:
                    with pytest.raises(gca.GCAError) as e:
                        cache.layout(f)
                    assert e.value.name == "GCA_ERR_STATE"
                    continue
                assert cache.layout(f) == want
        assert cache.evict() == sim.evict()
    cache.close()


def test_windowed_resets_give_fresh_tables():
    w = inputs.WINDOWED_VO.with_(L=1)
    cache, sim = _pair(w)
    fresh = None
    wins = w.windows()
    for idx in (0, 1, 2, len(wins) - 1):
        start, ln = wins[idx]
        cache.reset()
        sim.reset()
        assert cache.info().frames == 0
        walks = []
        for _ in range(ln):
            _step(cache, sim)
            walks.append(cache.layout())
            assert walks[-1] == sim.walk()
        if fresh is None:
            fresh = walks
        else:
            assert walks == fresh[:ln]        # page tables identical to a fresh cache's
    cache.close()


def test_capacity_and_state_errors():
    w = inputs.TINY
    cache, _ = _pair(w, max_frames=5)
    for t in range(5):
        cache.append(None, None)
        cache.evict()
    with pytest.raises(gca.GCAError) as e:
        cache.append(None, None)
    assert e.value.name == "GCA_ERR_CAPACITY"
    cache.close()

    w2 = inputs.TINY.with_(L=2)
    cache, _ = _pair(w2)
    with pytest.raises(gca.GCAError) as e:
        cache.append(None, None, layer=1)        # no open frame for layer 1
    assert e.value.name == "GCA_ERR_STATE"
    cache.append(None, None, layer=0)
    with pytest.raises(gca.GCAError) as e:
        cache.append(None, None, layer=0)        # layer 1 still misses frame 0
    assert e.value.name == "GCA_ERR_STATE"
    cache.append(None, None, layer=1)
    assert cache.append(None, None) == 1
    with pytest.raises(gca.GCAError) as e:
        cache.layout(3)                          # block larger than the stream
    assert e.value.name == "GCA_ERR_STATE"
    cache.close()


def test_attention_is_unsupported_without_a_device():
    import torch
    w = inputs.TINY
    cache, _ = _pair(w)
    cache.append(None, None)
    q = torch.zeros((1, w.Lq, w.H, w.D))
    out = torch.empty_like(q)
    for call in (lambda: cache.attend(0, q, out),
                 lambda: cache.attend_transient(0, q[0], q[0], q[0], out[0]),
                 lambda: cache.frame_attention(0, q[0], q[0], q[0], out[0])):
        with pytest.raises(gca.GCAError) as e:
            call()
        assert e.value.name == "GCA_ERR_UNSUPPORTED"
    assert cache.status() == 0
    cache.close()


def test_null_and_range_arguments_are_rejected():
    import ctypes
    w = inputs.TINY
    cache, _ = _pair(w)
    cache.append(None, None)
    L = gca.lib()
    n = ctypes.c_int32(0)
    e = gca.gca_page_entry_t(0, gca.GCA_PAGE_IMAGE, 0, 0, 16)
    assert gca.STATUS[L.gca_get_layout(cache.handle, 1, None, 0, None)] == "GCA_ERR_INVALID_ARG"
    assert gca.STATUS[L.gca_get_layout(cache.handle, 1, None, 4, ctypes.byref(n))] == "GCA_ERR_INVALID_ARG"
    assert gca.STATUS[L.gca_token_slot(cache.handle, 0, 0, None, None)] == "GCA_ERR_INVALID_ARG"
    assert gca.STATUS[L.gca_visible_prefix(cache.handle, None, 0, ctypes.byref(n))] == "GCA_ERR_INVALID_ARG"
    assert gca.STATUS[L.gca_visible_prefix(cache.handle, ctypes.byref(e), -1, ctypes.byref(n))] == \
        "GCA_ERR_INVALID_ARG"
    assert gca.STATUS[L.gca_get_info(None, None)] == "GCA_ERR_INVALID_ARG"
    assert gca.STATUS[L.gca_evict_to_summary(None, None)] == "GCA_ERR_INVALID_ARG"
    assert gca.STATUS[L.gca_reset(None)] == "GCA_ERR_INVALID_ARG"
    with pytest.raises(gca.GCAError) as err:
        cache.token_slot(1, 0)                      # frame not appended
    assert err.value.name == "GCA_ERR_INVALID_ARG"
    with pytest.raises(gca.GCAError) as err:
        cache.token_slot(0, w.Lq)                   # tau out of range
    assert err.value.name == "GCA_ERR_INVALID_ARG"
    with pytest.raises(gca.GCAError) as err:
        gca.Cache.for_workload(w, device=gca.GCA_HOST_ONLY, trajectory_memory=3)
    assert err.value.name == "GCA_ERR_INVALID_ARG"
    assert L.gca_cache_destroy(None) == 0            # null is accepted
    cache.close()


def test_walk_list_is_the_same_before_and_after_the_eviction():
    # gca_attend may run with the step's eviction still pending: for a single
    # query frame the walk list holds only the frames it may see, so it does
    # not change when the frame that left the window gives back its pages
    w = inputs.METRIC_518x378.with_(L=1)
    cache, sim = _pair(w)
    for t in range(200):
        assert cache.append(None, None) == sim.append()
        before = cache.layout()
        n = cache.evict()
        assert n == sim.evict() == (1 if t >= w.n + w.k else 0)
        assert cache.layout() == before == sim.walk()


def test_rope_configuration_is_checked():
    w = inputs.TINY
    for bad in ({"rope": 2}, {"rope": -1}, {"rope": gca.GCA_ROPE_3D, "rope_grid_w": -1},
                {"rope": gca.GCA_ROPE_3D, "rope_base": -5.0}):
        with pytest.raises(gca.GCAError) as e:
            gca.Cache.for_workload(w, device=gca.GCA_HOST_ONLY, **bad)
        assert e.value.name == "GCA_ERR_INVALID_ARG"
    c = gca.Cache.for_workload(w, device=gca.GCA_HOST_ONLY, rope=gca.GCA_ROPE_3D, rope_grid_w=4)
    assert c.append(None, None) == 0
