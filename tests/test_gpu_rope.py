"""GPU parity of the fused 3D rotary position encoding (gca_config_t.rope).

The library rotates K inside the append kernel as it stores it and rotates q
inside the attention kernels as they load it.  The oracle rotates the same
raw inputs with its explicit rotation matrices (oracle.gca.rope_frame: fp64,
then held in the workload dtype), and computes the attention of the rotated
vectors.  Tolerances are those of the other parity tests.
"""
import numpy as np
import pytest
import torch

from oracle import gca as ogca
from windowed_memory_attention_b200 import gca, inputs
from gca_stream_util import Mirror, attend, attend_transient, max_err, oracle_step, oracle_transient, pool_view

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}


def _rot(w, x, frame, grid_w):
    """Oracle rotation of one layer's frame tensor [S+M][H][D] (any device)."""
    return torch.from_numpy(ogca.rope_frame(x.float().cpu().numpy(), frame, S=w.S, grid_w=grid_w,
                                            dtype=w.dtype))


def _cache(w, grid_w, **extra):
    return gca.Cache.for_workload(w, rope=gca.GCA_ROPE_3D, rope_grid_w=grid_w, **extra)


@pytest.mark.parametrize("w", [inputs.TINY, inputs.TINY_BF16], ids=["f32", "bf16"])
def test_rope_stream_every_step(w):
    grid_w = 4                                   # 16 image tokens: a 4 x 4 patch grid
    cache = _cache(w, grid_w)
    mirror = Mirror(w, [0])
    errs = []
    for t in range(w.T):
        k, v, q = (inputs.draw(w, t, x) for x in "kvq")
        cache.append(k.cuda(), v.cuda())
        cache.evict()
        mirror.record(t, _rot(w, k[0], t, grid_w)[None], v, keep_full=True)
        out, lse = attend(cache, 0, q.cuda())
        qr = _rot(w, q[0], t, grid_w)[None].numpy()
        want, wlse = oracle_step(mirror, 0, qr, t)
        torch.cuda.synchronize()
        errs.append(max_err(out, want))
        assert errs[-1] <= TOL[w.dtype], t
        assert max_err(lse, wlse) <= TOL[w.dtype], t
    assert cache.status() == 0
    print(f"{w.name} rope: max |dO| {max(errs):.3e}")


@pytest.mark.parametrize("w", [inputs.TINY, inputs.TINY_BF16], ids=["f32", "bf16"])
def test_rope_keys_in_the_pool_are_the_rotated_keys(w):
    grid_w = 4
    cache = _cache(w, grid_w)
    frames = {}
    for t in range(8):
        k, v = inputs.draw(w, t, "k"), inputs.draw(w, t, "v")
        cache.append(k.cuda(), v.cuda())
        cache.evict()
        frames[t] = (_rot(w, k[0], t, grid_w), v[0])
    torch.cuda.synchronize()
    info = cache.info()
    shape = (w.L, info.num_pages, w.H, w.page_size, w.D)
    kp = pool_view(cache, "k", w.torch_dtype()).view(shape).float().cpu()
    vp = pool_view(cache, "v", w.torch_dtype()).view(shape).float().cpu()
    worst = 0.0
    for t, (kr, v) in frames.items():
        for tau in range(w.Lq):
            try:
                pid, slot = cache.token_slot(t, tau)
            except gca.GCAError:
                continue
            got = kp[0, pid, :, slot, :]
            # the kernel rotates in fp32 and rounds once to the cache dtype, the
            # oracle rotates in fp64 and rounds once: one unit in the last place
            # apart, or an fp32 rounding of the pair's norm where a component
            # nearly cancels
            pair = kr[tau].view(w.H, w.D // 2, 2)
            norm = torch.sqrt((pair ** 2).sum(-1, keepdim=True)).expand(-1, -1, 2).reshape(w.H, w.D)
            ulp = torch.abs(kr[tau]) * (2.0 ** -7 if w.dtype == "bf16" else 2.0 ** -23)
            allow = torch.maximum(ulp, norm * 2.0 ** -21) + 1e-30
            worst = max(worst, float((torch.abs(got - kr[tau]) / allow).max()))
            assert torch.equal(vp[0, pid, :, slot, :], v[tau].float())      # V is not rotated
    assert worst <= 1.0, worst


def test_rope_worked_example_shape():
    # 500 image tokens on a 25 x 20 grid, 16 heads, 4 image pages per frame
    w = inputs.WORKED_EXAMPLE.with_(T=40)
    grid_w = 25
    cache = _cache(w, grid_w)
    mirror = Mirror(w, [0])
    rows = [0, 1, 5, 6, 7, 127, 128, 255, 256, 383, 384, 505]
    for t in range(w.T):
        k, v = inputs.draw(w, t, "k", "cuda"), inputs.draw(w, t, "v", "cuda")
        cache.append(k, v)
        cache.evict()
        mirror.record(t, _rot(w, k[0], t, grid_w)[None], v, keep_full=t < w.n or t >= w.T - w.k)
    q = inputs.draw(w, w.T - 1, "q", "cuda")
    out, lse = attend(cache, 0, q)
    qr = _rot(w, q[0], w.T - 1, grid_w)[None].numpy()
    want, wlse = oracle_step(mirror, 0, qr, w.T - 1, rows=rows)
    torch.cuda.synchronize()
    assert max_err(out[0][rows], want[0]) <= TOL["bf16"]
    assert max_err(lse[0][rows], wlse[0]) <= TOL["bf16"]
    assert cache.status() == 0


@pytest.mark.parametrize("w", [inputs.TINY, inputs.TINY_BF16], ids=["f32", "bf16"])
def test_rope_non_keyframe_and_frame_attention(w):
    grid_w = 4
    cache = _cache(w, grid_w)
    mirror = Mirror(w, [0])
    T = 12
    for t in range(T):
        k, v = inputs.draw(w, t, "k"), inputs.draw(w, t, "v")
        cache.append(k.cuda(), v.cuda())
        cache.evict()
        mirror.record(t, _rot(w, k[0], t, grid_w)[None], v, keep_full=True)
    # a non-keyframe takes the latest keyframe's time index (T-1)
    qn, kn, vn = (inputs.draw(w, 500, x)[0] for x in "qkv")
    out, lse = attend_transient(cache, 0, qn.cuda(), kn.cuda(), vn.cuda())
    want, wlse = oracle_transient(mirror, 0, _rot(w, qn, T - 1, grid_w).numpy(),
                                  _rot(w, kn, T - 1, grid_w).numpy(), vn.float().numpy(), T - 1)
    torch.cuda.synchronize()
    assert max_err(out, want) <= TOL[w.dtype]
    assert max_err(lse, wlse) <= TOL[w.dtype]
    # intra-frame attention: every token of the frame, positions at t = 0
    outf = torch.empty_like(qn.cuda())
    lsef = torch.empty(qn.shape[:2], dtype=torch.float32, device="cuda")
    cache.frame_attention(0, qn.cuda(), kn.cuda(), vn.cuda(), outf, lsef)
    o, l = ogca.attention_np(_rot(w, qn, 0, grid_w).numpy(), _rot(w, kn, 0, grid_w).numpy(),
                             vn.float().numpy(), w.softmax_scale)
    torch.cuda.synchronize()
    assert max_err(outf, o) <= TOL[w.dtype]
    assert max_err(lsef, l) <= TOL[w.dtype]
    assert cache.status() == 0


def test_rope_changes_the_output():
    # the encoding is live: the same stream without it gives a different answer
    w = inputs.TINY_BF16
    outs = []
    for rope in (gca.GCA_ROPE_NONE, gca.GCA_ROPE_3D):
        cache = gca.Cache.for_workload(w, rope=rope, rope_grid_w=4)
        for t in range(10):
            cache.append(inputs.draw(w, t, "k", "cuda"), inputs.draw(w, t, "v", "cuda"))
            cache.evict()
        out, _ = attend(cache, 0, inputs.draw(w, 9, "q", "cuda"))
        torch.cuda.synchronize()
        outs.append(out.float())
    assert float((outs[0] - outs[1]).abs().max()) > 0.05
