"""GPU parity of the C-ABI library against the CPU oracle.

Every comparison runs the library's kernels through the C ABI on seeded inputs
and the oracle (oracle/) on the same values.  Tolerances: max |O_gpu - O_oracle|
<= 1e-4 for the fp32 cache, <= 2e-2 for bf16 inputs with fp32 accumulation;
page tables and pool bytes bit-exact.
"""
import math

import numpy as np
import pytest
import torch

from oracle.allocator import PageTableSim
from windowed_memory_attention_b200 import gca, inputs
from gca_stream_util import (Mirror, attend, attend_transient, max_err, needed_full, oracle_step,
                             oracle_transient, pool_view)

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}
LSE_TOL = {"f32": 1e-4, "bf16": 2e-2}


def _sim(w, **kw):
    return PageTableSim(M=w.M, S=w.S, P=w.page_size, n=w.n, k=w.k,
                        max_frames=kw.pop("max_frames", w.window_frames or w.T), **kw)


def _rows_sample(Lq, extra=0, seed=0):
    base = {0, 1, 5, 6, 7, 127, 128, 129, 255, 256, Lq // 2, Lq - 2, Lq - 1}
    rng = np.random.default_rng(seed)
    base |= set(rng.integers(0, Lq, size=extra).tolist())
    return sorted(r for r in base if 0 <= r < Lq)


# ----------------------------------------------------------------------------
# tiny workload: every step, full rows, both dtypes
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("w", [inputs.TINY, inputs.TINY_BF16], ids=["f32", "bf16"])
def test_tiny_stream_every_step(w):
    cache = gca.Cache.for_workload(w)
    sim = _sim(w)
    mirror = Mirror(w, [0])
    errs = []
    for t in range(w.T):
        k = inputs.draw(w, t, "k").cuda()
        v = inputs.draw(w, t, "v").cuda()
        q = inputs.draw(w, t, "q").cuda()
        assert cache.append(k, v) == t
        sim.append()
        mirror.record(t, k, v, keep_full=True)
        assert cache.evict() == sim.evict()
        assert cache.layout() == sim.walk()
        info = cache.info()
        assert info.resident_tokens == sim.resident_tokens()
        out, lse = attend(cache, 0, q)
        want, wlse = oracle_step(mirror, 0, q.float().cpu().numpy(), t)
        torch.cuda.synchronize()
        errs.append((max_err(out, want), max_err(lse, wlse)))
        assert errs[-1][0] <= TOL[w.dtype], t
        assert errs[-1][1] <= LSE_TOL[w.dtype], t
    assert cache.status() == 0
    print(f"{w.name}: max |dO| {max(e[0] for e in errs):.3e}, max |dlse| {max(e[1] for e in errs):.3e}")


MEMORY = {"summary": (gca.GCA_MEMORY_SUMMARY, 6, None), "camera": (gca.GCA_MEMORY_CAMERA, 1, None),
          "none_n0": (gca.GCA_MEMORY_NONE, 0, 0)}


@pytest.mark.parametrize("memory", list(MEMORY))
@pytest.mark.parametrize("w", [inputs.TINY, inputs.TINY_BF16], ids=["f32", "bf16"])
def test_append_writes_pool_bytes_bit_exact(w, memory):
    mode, keep, n = MEMORY[memory]
    if n is not None:
        w = w.with_(n=n)
    cache = gca.Cache.for_workload(w, trajectory_memory=mode)
    sim = _sim(w, keep=keep)
    frames = {}
    for t in range(w.T):
        k = inputs.draw(w, t, "k").cuda()
        v = inputs.draw(w, t, "v").cuda()
        cache.append(k, v)
        sim.append()
        assert cache.evict() == sim.evict()
        assert cache.layout() == sim.walk()
        frames[t] = (k[0].cpu(), v[0].cpu())
    torch.cuda.synchronize()
    info = cache.info()
    P, H, D = w.page_size, w.H, w.D
    for which, idx in (("k", 0), ("v", 1)):
        pool = pool_view(cache, which, w.torch_dtype()).view(w.L, info.num_pages, H, P, D).cpu()
        for t, kv in frames.items():
            for tau in range(w.Lq):
                try:
                    pid, slot = cache.token_slot(t, tau)
                except gca.GCAError as e:
                    assert e.name == "GCA_ERR_STATE" and tau >= keep   # left with the image pages
                    continue
                assert (pid, slot) == sim.slot_of(t, tau)
                got = pool[0, pid, :, slot, :]
                assert torch.equal(got.view(torch.int16 if w.dtype == "bf16" else torch.int32),
                                   kv[idx][tau].view(torch.int16 if w.dtype == "bf16" else torch.int32))


# ----------------------------------------------------------------------------
# multi-frame query blocks and the anchor block
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_anchor_block_then_stream(dtype):
    w = inputs.TINY.with_(dtype=dtype, T=14)
    cache = gca.Cache.for_workload(w, anchor_block=True, max_query_frames=w.n)
    sim = _sim(w, anchor_block=True, max_query_frames=w.n)
    mirror = Mirror(w, [0])
    qs = []
    for t in range(w.n):
        k, v = inputs.draw(w, t, "k").cuda(), inputs.draw(w, t, "v").cuda()
        cache.append(k, v)
        sim.append()
        mirror.record(t, k, v, keep_full=True)
        qs.append(inputs.draw(w, t, "q").cuda()[0])
    qb = torch.stack(qs)
    assert cache.layout(w.n) == sim.walk(w.n)
    out, lse = attend(cache, 0, qb, F=w.n)
    want, wlse = oracle_step(mirror, 0, qb.float().cpu().numpy(), w.n - 1, F=w.n, anchor_block=True)
    torch.cuda.synchronize()
    assert max_err(out, want) <= TOL[dtype]
    assert max_err(lse, wlse) <= LSE_TOL[dtype]
    for t in range(w.n, w.T):
        k, v, q = (inputs.draw(w, t, x).cuda() for x in "kvq")
        cache.append(k, v)
        sim.append()
        mirror.record(t, k, v, keep_full=True)
        assert cache.evict() == sim.evict()
        assert cache.layout() == sim.walk()
        out, lse = attend(cache, 0, q)
        want, wlse = oracle_step(mirror, 0, q.float().cpu().numpy(), t, anchor_block=True)
        torch.cuda.synchronize()
        assert max_err(out, want) <= TOL[dtype], t


@pytest.mark.parametrize("F", [2, 3])
def test_multi_frame_blocks(F):
    w = inputs.TINY_BF16.with_(T=20)
    cache = gca.Cache.for_workload(w, max_query_frames=F)
    sim = _sim(w, max_query_frames=F)
    mirror = Mirror(w, [0])
    t = 0
    while t + F <= w.T:
        qs = []
        for b in range(F):
            k, v = inputs.draw(w, t + b, "k").cuda(), inputs.draw(w, t + b, "v").cuda()
            cache.append(k, v)
            sim.append()
            mirror.record(t + b, k, v, keep_full=True)
            qs.append(inputs.draw(w, t + b, "q").cuda()[0])
        last = t + F - 1
        assert cache.layout(F) == sim.walk(F)
        qb = torch.stack(qs)
        out, lse = attend(cache, 0, qb, F=F)
        want, wlse = oracle_step(mirror, 0, qb.float().cpu().numpy(), last, F=F)
        torch.cuda.synchronize()
        assert max_err(out, want) <= TOL["bf16"], last
        assert max_err(lse, wlse) <= LSE_TOL["bf16"], last
        assert cache.evict() == sim.evict()
        t += F


# ----------------------------------------------------------------------------
# host pointers (the end-to-end path), reset, errors
# ----------------------------------------------------------------------------
def test_host_pointer_path_matches_device_path():
    w = inputs.TINY_BF16
    a = gca.Cache.for_workload(w)
    b = gca.Cache.for_workload(w)
    for t in range(12):
        k, v, q = (inputs.draw(w, t, x) for x in "kvq")
        a.append(k.cuda(), v.cuda())
        b.append(k.pin_memory(), v)                  # pinned and pageable host inputs
        a.evict()
        b.evict()
        out_d, lse_d = attend(a, 0, q.cuda())
        out_h = torch.empty_like(q).pin_memory()
        lse_h = torch.empty(q.shape[:3], dtype=torch.float32).pin_memory()
        b.attend(0, q.pin_memory(), out_h, lse_h)
        torch.cuda.synchronize()
        assert torch.equal(out_d.cpu(), out_h)
        assert torch.equal(lse_d.cpu(), lse_h)


def test_all_host_calls_on_a_side_stream_match_device_path():
    """Calls whose pointers are all host memory run on the library's stream and
    overlap their copies back; the caller's stream still waits for each call,
    so synchronising that stream alone makes the outputs readable.  Device-
    pointer calls interleaved with them keep the cache's order."""
    w = inputs.TINY_BF16.with_(L=3)
    a = gca.Cache.for_workload(w)
    b = gca.Cache.for_workload(w)
    side = torch.cuda.Stream()
    for t in range(14):
        k, v, q = (inputs.draw(w, t, x) for x in "kvq")
        a.append(k.cuda(), v.cuda())
        a.evict()
        mixed = t % 5 == 3            # every fifth frame goes through device pointers
        with torch.cuda.stream(side):
            if mixed:
                b.append(k.cuda(), v.cuda(), stream=side)
            else:
                b.append(k.pin_memory(), v.pin_memory(), stream=side)
        b.evict()
        outs_d = [attend(a, l, q[l:l + 1].cuda()) for l in range(w.L)]
        torch.cuda.synchronize()
        q_h = q.pin_memory()
        out_h = [torch.empty_like(q[0:1]).pin_memory() for _ in range(w.L)]
        lse_h = [torch.empty(q[0:1].shape[:3], dtype=torch.float32).pin_memory() for _ in range(w.L)]
        for l in range(w.L):
            if mixed and l == 1:
                o_dev = torch.empty_like(q[0:1], device="cuda")
                l_dev = torch.empty(q[0:1].shape[:3], dtype=torch.float32, device="cuda")
                b.attend(l, q_h[l:l + 1], o_dev, l_dev, stream=side)
                with torch.cuda.stream(side):
                    out_h[l].copy_(o_dev, non_blocking=True)
                    lse_h[l].copy_(l_dev, non_blocking=True)
            else:
                b.attend(l, q_h[l:l + 1], out_h[l], lse_h[l], stream=side)
        side.synchronize()
        for l in range(w.L):
            assert torch.equal(outs_d[l][0].cpu(), out_h[l]), (t, l)
            assert torch.equal(outs_d[l][1].cpu(), lse_h[l]), (t, l)
    assert b.status() == 0


def test_reset_gives_fresh_tables_and_outputs():
    w = inputs.TINY_BF16
    c = gca.Cache.for_workload(w)
    fresh = gca.Cache.for_workload(w)

    def run(cache, start, n):
        outs = []
        for t in range(start, start + n):
            k, v, q = (inputs.draw(w, t, x).cuda() for x in "kvq")
            cache.append(k, v)
            cache.evict()
            outs.append((cache.layout(), attend(cache, 0, q)[0]))
        return outs

    run(c, 0, 20)
    c.reset()
    info = c.info()
    assert info.frames == 0 and info.full_frames == 0 and info.resident_tokens == 0
    a = run(c, 100, 15)
    b = run(fresh, 100, 15)
    torch.cuda.synchronize()
    for (la, oa), (lb, ob) in zip(a, b):
        assert la == lb
        assert torch.equal(oa, ob)


def test_state_and_argument_errors():
    w = inputs.TINY_BF16.with_(L=2)
    c = gca.Cache.for_workload(w, max_frames=3)
    q = inputs.draw(w, 0, "q").cuda()
    out = torch.empty_like(q[0:1].contiguous())
    with pytest.raises(gca.GCAError) as e:
        c.attend(0, q[0:1].contiguous(), out)         # nothing appended
    assert e.value.name == "GCA_ERR_STATE"
    k, v = inputs.draw(w, 0, "k").cuda(), inputs.draw(w, 0, "v").cuda()
    with pytest.raises(gca.GCAError) as e:
        c.append(k[1].contiguous(), v[1].contiguous(), layer=1)   # layer 1 before frame opened
    assert e.value.name == "GCA_ERR_STATE"
    c.append(k[0].contiguous(), v[0].contiguous(), layer=0)
    with pytest.raises(gca.GCAError) as e:
        c.append(k[0].contiguous(), v[0].contiguous(), layer=0)   # layer 1 still misses frame 0
    assert e.value.name == "GCA_ERR_STATE"
    with pytest.raises(gca.GCAError) as e:
        c.attend(1, q[1:2].contiguous(), out)        # layer 1 has not appended frame 0
    assert e.value.name == "GCA_ERR_STATE"
    c.append(k[1].contiguous(), v[1].contiguous(), layer=1)
    c.attend(1, q[1:2].contiguous(), out)
    with pytest.raises(gca.GCAError) as e:
        c.attend(0, q[0:1].contiguous(), out, num_query_frames=2)   # above max_query_frames
    assert e.value.name == "GCA_ERR_INVALID_ARG"
    with pytest.raises(gca.GCAError) as e:
        c.attend(5, q[0:1].contiguous(), out)
    assert e.value.name == "GCA_ERR_INVALID_ARG"
    c.append(k, v)
    c.append(k, v)
    with pytest.raises(gca.GCAError) as e:
        c.append(k, v)                               # max_frames = 3
    assert e.value.name == "GCA_ERR_CAPACITY"
    assert c.info().frames == 3
    with pytest.raises(gca.GCAError) as e:
        gca.Cache(num_layers=1, num_heads=2, image_tokens=16, num_anchor=3, window=4,
                  max_frames=8, head_dim=128)
    assert e.value.name == "GCA_ERR_UNSUPPORTED"
    with pytest.raises(gca.GCAError) as e:
        gca.Cache(num_layers=0, num_heads=2, image_tokens=16, num_anchor=3, window=4, max_frames=8)
    assert e.value.name == "GCA_ERR_INVALID_ARG"
    r = gca.lib().gca_attend(c.handle, 0, None, 1, None, None, None)
    assert gca.STATUS[r] == "GCA_ERR_INVALID_ARG"
    assert c.status() == 0


def test_page_size_64():
    w = inputs.TINY_BF16.with_(M=150, page_size=64, T=12)
    cache = gca.Cache.for_workload(w)
    sim = _sim(w)
    mirror = Mirror(w, [0])
    for t in range(w.T):
        k, v, q = (inputs.draw(w, t, x).cuda() for x in "kvq")
        cache.append(k, v)
        sim.append()
        mirror.record(t, k, v, keep_full=True)
        assert cache.evict() == sim.evict()
        assert cache.layout() == sim.walk()
        out, lse = attend(cache, 0, q)
        want, _ = oracle_step(mirror, 0, q.float().cpu().numpy(), t)
        torch.cuda.synchronize()
        assert max_err(out, want) <= TOL["bf16"], t


# ----------------------------------------------------------------------------
# trajectory-memory variants: camera token only; none (sliding window, n = 0)
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("memory", ["camera", "none_n0"])
@pytest.mark.parametrize("w", [inputs.TINY, inputs.TINY_BF16], ids=["f32", "bf16"])
def test_memory_variant_stream_every_step(w, memory):
    mode, keep, n = MEMORY[memory]
    if n is not None:
        w = w.with_(n=n)
    cache = gca.Cache.for_workload(w, trajectory_memory=mode)
    sim = _sim(w, keep=keep)
    mirror = Mirror(w, [0])
    for t in range(w.T):
        k, v, q = (inputs.draw(w, t, x).cuda() for x in "kvq")
        assert cache.append(k, v) == t
        sim.append()
        mirror.record(t, k, v, keep_full=True)
        assert cache.evict() == sim.evict()
        assert cache.layout() == sim.walk()
        assert cache.info().resident_tokens == sim.resident_tokens()
        out, lse = attend(cache, 0, q[0:1].contiguous())
        want, wlse = oracle_step(mirror, 0, q[0:1].float().cpu().numpy(), t, keep=keep)
        torch.cuda.synchronize()
        assert max_err(out[0], want[0]) <= TOL[w.dtype], t
        assert max_err(lse[0], wlse[0]) <= LSE_TOL[w.dtype], t
    assert cache.status() == 0


# ----------------------------------------------------------------------------
# non-keyframe steps: only keyframes enter the cache
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("interval", [2, 3])
@pytest.mark.parametrize("w", [inputs.TINY, inputs.TINY_BF16], ids=["f32", "bf16"])
def test_keyframe_interval_stream(w, interval):
    """Video frames 0..T-1; keyframes (the n scale frames, then every
    interval-th frame) are appended and evicted, the others attend through
    gca_attend_transient and leave the page table untouched."""
    cache = gca.Cache.for_workload(w)
    sim = _sim(w)
    mirror = Mirror(w, range(w.L))
    kid = -1
    n_trans = 0
    for x in range(w.T):
        k = inputs.draw(w, x, "k").cuda()
        v = inputs.draw(w, x, "v").cuda()
        q = inputs.draw(w, x, "q").cuda()
        if x < w.n or (x - w.n) % interval == 0:
            kid += 1
            assert cache.append(k, v) == kid
            sim.append()
            mirror.record(kid, k, v, keep_full=True)
            assert cache.evict() == sim.evict()
            out, _ = attend(cache, 0, q[0:1].contiguous())
            want, _ = oracle_step(mirror, 0, q[0:1].float().cpu().numpy(), kid)
            torch.cuda.synchronize()
            assert max_err(out[0], want[0]) <= TOL[w.dtype], x
            continue
        launches = cache.info().kernel_launches
        for l in range(w.L):
            out, lse = attend_transient(cache, l, q[l], k[l], v[l])
            want, wlse = oracle_transient(mirror, l, q[l].float().cpu().numpy(),
                                          k[l].float().cpu().numpy(), v[l].float().cpu().numpy(), kid)
            torch.cuda.synchronize()
            assert max_err(out, want) <= TOL[w.dtype], (x, l)
            assert max_err(lse, wlse) <= LSE_TOL[w.dtype], (x, l)
        n_trans += 1
        # nothing was kept: same frame count, tables and resident tokens
        assert cache.layout() == sim.walk()
        info = cache.info()
        assert info.frames == kid + 1 and info.resident_tokens == sim.resident_tokens()
        assert info.kernel_launches > launches
    assert n_trans > 0 and cache.status() == 0


@pytest.mark.parametrize("w", [inputs.TINY, inputs.TINY_BF16], ids=["f32", "bf16"])
def test_transient_before_any_keyframe_and_host_pointers(w):
    """With an empty cache a non-keyframe reads only its own tokens; host
    tensors give the same result as device tensors."""
    cache = gca.Cache.for_workload(w)
    mirror = Mirror(w, [0])
    q, k, v = (inputs.draw(w, 5, x)[0] for x in "qkv")
    out, lse = attend_transient(cache, 0, q.cuda(), k.cuda(), v.cuda())
    want, wlse = oracle_transient(mirror, 0, q.float().numpy(), k.float().numpy(), v.float().numpy(), -1)
    torch.cuda.synchronize()
    assert max_err(out, want) <= TOL[w.dtype]
    assert max_err(lse, wlse) <= LSE_TOL[w.dtype]
    out_h = torch.empty_like(q).pin_memory()
    lse_h = torch.empty(q.shape[:2], dtype=torch.float32).pin_memory()
    cache.attend_transient(0, q.pin_memory(), k.pin_memory(), v.pin_memory(), out_h, lse_h)
    torch.cuda.synchronize()
    assert torch.equal(out_h, out.cpu()) and torch.equal(lse_h, lse.cpu())
    assert cache.info().frames == 0


def _misaligned(x: torch.Tensor) -> torch.Tensor:
    """The same values at an address 8 bytes past a 16-byte boundary."""
    flat = torch.empty(x.numel() + 4, dtype=x.dtype, device=x.device)
    view = flat[4:].view(x.shape)
    view.copy_(x)
    assert view.data_ptr() % 16 == 8
    return view


@pytest.mark.parametrize("w", [inputs.TINY_BF16, inputs.METRIC_518x378.with_(L=1)], ids=["bf16", "518x378"])
def test_frame_tokens_read_in_place_and_misaligned_tensors_refused(w):
    """bf16 K/V of the query frame are read in place by the attention kernel
    (a 3D tensor map over [S+M][H][D]): one launch per non-keyframe or
    intra-frame call (their values against the oracle: the transient and
    intra-frame tests).  A device tensor off a 16-byte boundary is refused
    before anything is launched or changed."""
    cache = gca.Cache.for_workload(w)
    for t in range(w.n + 2):
        cache.append(inputs.draw(w, t, "k").cuda(), inputs.draw(w, t, "v").cuda())
        cache.evict()
    q, k, v = (inputs.draw(w, w.n + 7, x)[0].cuda() for x in "qkv")
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:2], dtype=torch.float32, device=q.device)
    for call in (cache.attend_transient, cache.frame_attention):
        n0 = cache.info().kernel_launches
        call(0, q, k, v, out, lse)
        assert cache.info().kernel_launches - n0 == 1
    torch.cuda.synchronize()
    layout, n0 = cache.layout(), cache.info().kernel_launches
    bad = [(_misaligned(q), k, v), (q, _misaligned(k), v), (q, k, _misaligned(v))]
    for qq, kk, vv in bad:
        for call in (cache.attend_transient, cache.frame_attention):
            with pytest.raises(gca.GCAError) as e:
                call(0, qq, kk, vv, out, lse)
            assert e.value.name == "GCA_ERR_INVALID_ARG"
    kw, vw = inputs.draw(w, w.n + 2, "k").cuda(), inputs.draw(w, w.n + 2, "v").cuda()
    for refused in (lambda: cache.attend(0, _misaligned(q)[None], out[None]),
                    lambda: cache.attend(0, q[None], _misaligned(out)[None]),
                    lambda: cache.append(_misaligned(kw), vw),
                    lambda: cache.append(kw, _misaligned(vw))):
        with pytest.raises(gca.GCAError) as e:
            refused()
        assert e.value.name == "GCA_ERR_INVALID_ARG"
    assert cache.info().kernel_launches == n0 and cache.layout() == layout
    assert cache.info().frames == w.n + 2
    cache.append(kw, vw)                    # the cache goes on as before
    assert cache.status() == 0


# ----------------------------------------------------------------------------
# intra-frame attention (the layers that alternate with GCA)
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("w", [inputs.TINY, inputs.TINY_BF16, inputs.METRIC_518x378.with_(L=2)],
                         ids=["f32", "bf16", "518x378"])
def test_frame_attention_is_dense_attention_within_the_frame(w):
    """Every token attends to the frame's own tokens only; the cache's state is
    neither read nor changed (it holds other frames here)."""
    cache = gca.Cache.for_workload(w, max_frames=8)
    sim = _sim(w, max_frames=8)
    for t in range(3):
        cache.append(inputs.draw(w, t, "k", "cuda"), inputs.draw(w, t, "v", "cuda"))
        sim.append()
        cache.evict()
        sim.evict()
    mirror = Mirror(w, [0])
    rows = None if w.Lq <= 64 else _rows_sample(w.Lq, extra=8, seed=9)
    for l in range(w.L):
        q, k, v = (inputs.draw(w, 100 + l, x, "cuda", layers=[l])[0] for x in "qkv")
        out = torch.empty_like(q)
        lse = torch.empty(q.shape[:2], dtype=torch.float32, device="cuda")
        cache.frame_attention(l, q, k, v, out, lse)
        want, wlse = oracle_transient(mirror, l, q.float().cpu().numpy(), k.float().cpu().numpy(),
                                      v.float().cpu().numpy(), -1, rows=rows)
        torch.cuda.synchronize()
        got, gl = (out, lse) if rows is None else (out[rows], lse[rows])
        assert max_err(got, want) <= TOL[w.dtype], l
        assert max_err(gl, wlse) <= LSE_TOL[w.dtype], l
    assert cache.layout() == sim.walk() and cache.info().frames == 3 and cache.status() == 0


@pytest.mark.parametrize("w", [inputs.TINY, inputs.TINY_BF16, inputs.METRIC_518x378.with_(L=1)],
                         ids=["f32", "bf16", "518x378"])
def test_frame_attention_batch_is_per_frame_dense_attention(w):
    """F frames in one call: frame f's tokens attend to frame f's tokens only.
    bf16 device tensors go in one launch (one CTA per frame, tile pair and
    head); its output equals the single-frame call's bit for bit (same split:
    a frame's heads are short walks, never split) and the oracle's within the
    tolerance.  fp32 and host tensors take one call per frame."""
    cache = gca.Cache.for_workload(w, max_frames=8)
    mirror = Mirror(w, [0])
    F = 5 if w.Lq <= 64 else 3
    rows = None if w.Lq <= 64 else _rows_sample(w.Lq, extra=4, seed=11)
    q, k, v = (torch.stack([inputs.draw(w, 200 + f, x, "cuda")[0] for f in range(F)]) for x in "qkv")
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    n0 = cache.info().kernel_launches
    cache.frame_attention_batch(0, q, k, v, out, lse)
    launches = cache.info().kernel_launches - n0
    assert launches == (1 if w.dtype == "bf16" else 2 * F)       # fp32: copy + attention per frame
    for f in range(F):
        o1 = torch.empty_like(q[f])
        l1 = torch.empty(q.shape[1:3], dtype=torch.float32, device="cuda")
        cache.frame_attention(0, q[f], k[f], v[f], o1, l1)
        want, wlse = oracle_transient(mirror, 0, q[f].float().cpu().numpy(), k[f].float().cpu().numpy(),
                                      v[f].float().cpu().numpy(), -1, rows=rows)
        torch.cuda.synchronize()
        assert torch.equal(out[f], o1) and torch.equal(lse[f], l1), f
        got, gl = (out[f], lse[f]) if rows is None else (out[f][rows], lse[f][rows])
        assert max_err(got, want) <= TOL[w.dtype], f
        assert max_err(gl, wlse) <= LSE_TOL[w.dtype], f
    # host tensors: staged one frame per launch, same values
    out_h = torch.empty_like(q, device="cpu").pin_memory()
    cache.frame_attention_batch(0, q.cpu().pin_memory(), k.cpu().pin_memory(), v.cpu().pin_memory(), out_h)
    torch.cuda.synchronize()
    assert torch.equal(out_h, out.cpu())
    assert cache.info().frames == 0 and cache.status() == 0


# ----------------------------------------------------------------------------
# the larger workloads
# ----------------------------------------------------------------------------
def _stream(w, cache, sim, mirror, T, checks, layers_to_check, rows, frame0=0, reset=False,
            transient=False):
    """Stream frames frame0..frame0+T-1 (local indices 0..T-1); at each local
    step in `checks` compare sampled rows of the listed layers with the oracle
    (and, with `transient`, a non-keyframe's attention at that state).  `rows`
    is a list of token rows, None for every row, or a dict layer -> either."""
    dev = "cuda"
    if reset:
        cache.reset()
        sim.reset()
    heads = mirror.heads
    results = []
    for t in range(T):
        g = frame0 + t
        k = inputs.draw(w, g, "k", dev)
        v = inputs.draw(w, g, "v", dev)
        cache.append(k, v)
        sim.append()
        keep_full = any(t <= c and (t < w.n or t >= c - w.k + 1) for c in checks)
        mirror.record(t, k, v, keep_full=keep_full)
        assert cache.evict() == sim.evict()
        if t in checks:
            assert cache.layout() == sim.walk()
            q = inputs.draw(w, g, "q", dev)
            for l in layers_to_check:
                lrows = rows.get(l) if isinstance(rows, dict) else rows
                sel = slice(None) if lrows is None else lrows
                out, lse = attend(cache, l, q[l:l + 1].contiguous())
                torch.cuda.synchronize()
                want, wlse = oracle_step(mirror, l, q[l:l + 1].float().cpu().numpy(), t, rows=lrows)
                got, gl = out[0][sel], lse[0][sel]
                if heads is not None:
                    got, gl = got[:, heads], gl[:, heads]
                e = max_err(got, want[0])
                el = max_err(gl, wlse[0])
                results.append((t, l, e, el))
                assert e <= TOL["bf16"], (t, l, e)
                assert el <= LSE_TOL["bf16"], (t, l, el)
                assert torch.isfinite(out).all()
                if transient:
                    # a non-keyframe (tensors of a frame outside the stream)
                    qt, kt, vt = (inputs.draw(w, frame0 + T + 1, x, dev, layers=[l])[0] for x in "qkv")
                    out, lse = attend_transient(cache, l, qt, kt, vt)
                    torch.cuda.synchronize()
                    want, wlse = oracle_transient(mirror, l, qt.float().cpu().numpy(), kt.float().cpu().numpy(),
                                                  vt.float().cpu().numpy(), t, rows=lrows)
                    got, gl = out[sel], lse[sel]
                    if heads is not None:
                        got, gl = got[:, heads], gl[:, heads]
                    e = max_err(got, want)
                    results.append((t, l, "transient", e))
                    assert e <= TOL["bf16"], (t, l, "transient", e)
                    assert max_err(gl, wlse) <= LSE_TOL["bf16"], (t, l, "transient")
                    assert cache.layout() == sim.walk()
            mirror.drop_full(set(f for f in range(t + 1) if f < w.n) |
                             set(f for c in checks if c > t for f in range(max(0, c - w.k + 1), t + 1)))
    assert cache.status() == 0
    return results


def test_worked_example_to_T10000():
    w = inputs.WORKED_EXAMPLE
    cache = gca.Cache.for_workload(w)
    sim = _sim(w)
    mirror = Mirror(w, [0])
    rows = _rows_sample(w.Lq, extra=12)
    res = _stream(w, cache, sim, mirror, w.T, {99, 999, 9999}, [0], rows, transient=True)
    assert cache.info().resident_tokens == 500 * 19 + 6 * 10000
    print("worked example max errors", res)


def test_metric_workload_T10000_all_layers():
    # layer 0 in full (all 1005 rows x 16 heads) at T=10000, layer 23 on sampled rows
    w = inputs.METRIC_518x378
    cache = gca.Cache.for_workload(w)
    sim = _sim(w)
    mirror = Mirror(w, [0, 23])
    rows = {0: None, 23: _rows_sample(w.Lq, extra=8, seed=3)}
    res = _stream(w, cache, sim, mirror, w.T, {9999}, [0, 23], rows, transient=True)
    assert cache.info().resident_tokens == 999 * 67 + 6 * 10000
    # every layer's output at T=10000 is finite and its lse lies within the
    # bounds softmax attention allows: ln(#keys) - max|s| <= lse <= ln(#keys) + max|s|
    q = inputs.draw(w, w.T - 1, "q", "cuda")
    for l in range(w.L):
        out, lse = attend(cache, l, q[l:l + 1].contiguous())
        assert torch.isfinite(out).all() and torch.isfinite(lse).all()
        assert float(lse.min()) > math.log(126933) - 20 and float(lse.max()) < math.log(126933) + 20
    print("metric workload max errors", res)


def test_windowed_vo_full_stream():
    """The windowed (VO) workload as defined: 179 windows of 128 frames
    overlapping by 16 over 20,000 frames (22,848 frames processed), a reset at
    each window start, the window's first n frames its anchors.  Page tables
    match the simulator at every checked step of every window; sampled rows of
    two heads match the oracle at steps 0, 2, 66 and the window's last step."""
    w = inputs.WINDOWED_VO
    wins = w.windows()
    assert len(wins) == 179 and sum(ln for _, ln in wins) == 22848
    cache = gca.Cache.for_workload(w)
    sim = _sim(w)
    rows = _rows_sample(w.Lq, extra=2, seed=5)
    processed = 0
    for idx, (start, ln) in enumerate(wins):
        mirror = Mirror(w, [0], heads=[idx % w.H, (idx * 7 + 3) % w.H])
        checks = {c for c in (0, 2, 66, ln - 1) if c < ln}
        _stream(w, cache, sim, mirror, ln, checks, [0], rows, frame0=start, reset=True)
        processed += ln
        assert cache.info().frames == ln
    assert processed == 22848


def test_dense_causal_limit_T1000():
    w = inputs.DENSE_CAUSAL
    cache = gca.Cache.for_workload(w)
    sim = _sim(w)
    heads = [0, 9]
    mirror = Mirror(w, [0], heads=heads)
    rows = [0, 5, 6, 500, 1004]
    res = _stream(w, cache, sim, mirror, w.T, {999}, [0], rows)
    assert cache.info().resident_tokens == 1005 * 1000
    print("dense limit errors", res)


def test_bounded_wait_reports_instead_of_hanging():
    """A kernel wait that can never complete gives up after its deadline,
    raises the status word, and leaves the context usable: the next calls
    run and still match the oracle."""
    w = inputs.TINY_BF16
    cache = gca.Cache.for_workload(w)
    assert gca.gca_selftest_bounded_wait(cache.handle, 100) == 1
    k, v, q = (inputs.draw(w, 0, x).cuda() for x in "kvq")
    with pytest.raises(gca.GCAError) as e:
        cache.append(k, v)                      # the raised status word is reported
    assert e.value.name == "GCA_ERR_DEVICE_CHECK"
    assert cache.status(clear=True) == 1
    mirror = Mirror(w, [0])
    cache.append(k, v)
    mirror.record(0, k, v, keep_full=True)
    out, _ = attend(cache, 0, q)
    want, _ = oracle_step(mirror, 0, q.float().cpu().numpy(), 0)
    torch.cuda.synchronize()
    assert max_err(out, want) <= TOL["bf16"]
    assert cache.status() == 0
