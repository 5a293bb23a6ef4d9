"""The allocation-free attention entry point (gca_attend_pages_noalloc).

It exists for callers that cannot call cudaMalloc — a framework whose caching
allocator owns device memory, or a real-time loop that must not make a call
that can synchronise the device.  The test builds a cache with the normal
API, then runs the same attention through gca_attend and through the
allocation-free entry point (twice in a row, since every call reuses the same
static scratch array) and compares the outputs within the bf16 tolerance of
the parity tests.  This file sorts last so that a run stopping at the first
failure has already run every other test.
"""
import ctypes

import pytest
import torch

from windowed_memory_attention_b200 import gca, inputs

pytestmark = pytest.mark.gpu

TOL = 2e-2


def _stream(w, frames, F=1, **extra):
    cache = gca.Cache.for_workload(w, max_query_frames=F, **extra)
    for t in range(frames):
        k, v = inputs.draw(w, t, "k", "cuda"), inputs.draw(w, t, "v", "cuda")
        cache.append(k, v)
        if t < frames - F:
            cache.evict()
    return cache


def _entries(cache, F):
    lay = cache.layout(F)
    arr = (gca.gca_page_entry_t * len(lay))(*[gca.gca_page_entry_t(*e) for e in lay])
    return arr, len(lay)


KEPT = {gca.GCA_MEMORY_SUMMARY: None, gca.GCA_MEMORY_CAMERA: 1, gca.GCA_MEMORY_NONE: 0}


def _noalloc(cache, w, layer, q, F, walk, nwalk, num_pages=None, **extra):
    info = cache.info()
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    kept = KEPT[extra.get("trajectory_memory", gca.GCA_MEMORY_SUMMARY)]
    gca.gca_attend_pages_noalloc(
        info.k_pool, info.v_pool, num_layers=w.L,
        num_pages=info.num_pages if num_pages is None else num_pages, num_heads=w.H,
        page_size=w.page_size, layer=layer, walk=walk, nwalk=nwalk, q=q, num_query_frames=F,
        tokens_per_frame=w.Lq, first_query_frame=info.frames - F, num_anchor=w.n, window=w.k,
        summary_tokens=w.S if kept is None else kept, anchor_block=extra.get("anchor_block", False),
        softmax_scale=w.softmax_scale, out=out, lse=lse)
    return out, lse


@pytest.mark.parametrize("case", ["tiny", "split_heads", "block3_device_walk", "camera_only",
                                  "sliding_window"])
def test_noalloc_matches_gca_attend_on_two_calls(case):
    if case == "tiny":
        w, frames, F, layer, extra = inputs.TINY_BF16, 20, 1, 0, {}
    elif case == "camera_only":
        # one kept special token per frame (the camera token)
        w, frames, F, layer, extra = inputs.TINY_BF16, 20, 1, 0, {"trajectory_memory": gca.GCA_MEMORY_CAMERA}
    elif case == "sliding_window":
        # nothing kept and no anchors: the summary-token count is 0
        w, frames, F, layer, extra = inputs.TINY_BF16.with_(n=0), 20, 1, 0, {"trajectory_memory": gca.GCA_MEMORY_NONE}
    elif case == "split_heads":
        # 546 walk entries x 16 heads over 37 workers: heads are split, so the
        # partials and their counters go through the static scratch
        w, frames, F, layer, extra = inputs.METRIC_518x378.with_(L=2, T=200), 200, 1, 1, {}
    else:
        w, frames, F, layer, extra = inputs.TINY_BF16.with_(T=12), 3, 3, 0, {"anchor_block": True}
    cache = _stream(w, frames, F, **extra)
    qs = [inputs.draw(w, t, "q", "cuda")[layer] for t in range(frames - F, frames)]
    q = torch.stack(qs).contiguous()
    ref = torch.empty_like(q)
    ref_lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    cache.attend(layer, q, ref, ref_lse, num_query_frames=F)
    walk, nwalk = _entries(cache, F)
    if case == "block3_device_walk":
        dev_walk = torch.tensor([[e.page_id, e.kind, e.frame, e.first, e.n_valid] for e in walk],
                                dtype=torch.int32, device="cuda")
        walk = dev_walk.data_ptr()
    for call in range(2):
        out, lse = _noalloc(cache, w, layer, q, F, walk, nwalk, **extra)
        torch.cuda.synchronize()
        assert torch.isfinite(out.float()).all()
        assert (out.float() - ref.float()).abs().max().item() <= TOL, call
        assert (lse - ref_lse).abs().max().item() <= TOL, call
    assert cache.status() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    w = inputs.TINY_BF16
    cache = _stream(w, 4)
    info = cache.info()
    q = torch.zeros((1, w.Lq, w.H, w.D), dtype=torch.bfloat16, device="cuda")
    walk, nwalk = _entries(cache, 1)
    with pytest.raises(gca.GCAError) as e:
        # 40000 query frames -> ceil(40000*22/128) * 2 heads partial tiles > 512
        gca.gca_attend_pages_noalloc(
            info.k_pool, info.v_pool, num_layers=1, num_pages=info.num_pages, num_heads=w.H,
            page_size=w.page_size, layer=0, walk=walk, nwalk=nwalk, q=q, num_query_frames=40000,
            tokens_per_frame=w.Lq, first_query_frame=0, num_anchor=w.n, window=w.k,
            summary_tokens=w.S, anchor_block=False, softmax_scale=w.softmax_scale, out=q)
    assert e.value.name == "GCA_ERR_CAPACITY"


def test_noalloc_rejects_pools_smaller_than_the_sizes_say():
    # a num_pages past the pools' allocation is refused before any launch
    w = inputs.TINY_BF16
    cache = _stream(w, 6)
    info = cache.info()
    q = inputs.draw(w, 5, "q", "cuda")
    walk, nwalk = _entries(cache, 1)
    with pytest.raises(gca.GCAError) as e:
        _noalloc(cache, w, 0, q, 1, walk, nwalk, num_pages=info.num_pages * 1000)
    assert e.value.name == "GCA_ERR_INVALID_ARG"
    torch.cuda.synchronize()
    assert cache.status() == 0


def test_noalloc_rejects_bad_host_walk_entries():
    w = inputs.TINY_BF16
    cache = _stream(w, 6)
    info = cache.info()
    q = inputs.draw(w, 5, "q", "cuda")
    for field, value in (("page_id", info.num_pages), ("page_id", -1), ("n_valid", w.page_size + 1),
                         ("kind", 7)):
        walk, nwalk = _entries(cache, 1)
        setattr(walk[nwalk - 1], field, value)
        with pytest.raises(gca.GCAError) as e:
            _noalloc(cache, w, 0, q, 1, walk, nwalk)
        assert e.value.name == "GCA_ERR_INVALID_ARG", (field, value)
    # the entries as the cache lists them still work
    walk, nwalk = _entries(cache, 1)
    out, _ = _noalloc(cache, w, 0, q, 1, walk, nwalk)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
