"""The seeded input recipe (CPU only).

The seed mixer is checked against the published SplitMix64 sequence, the
workload shapes against the pages' numbers (518x378 at patch 14 gives 999
image tokens; windows of 128 frames overlapping by 16 over 20000 frames), and
the draw's properties that every parity test relies on: determinism, distinct
streams per frame / tensor / layer, rounding to the workload dtype, and the
lognormal key norms shared by the heads of a token.
"""
import math

import torch

from windowed_memory_attention_b200 import inputs


def test_splitmix64_matches_the_published_sequence():
    # Steele, Lea, Flood (OOPSLA 2014) / Vigna's reference splitmix64: the first
    # three outputs of the generator started at state 0
    state, outs = 0, []
    for _ in range(3):
        outs.append(inputs.splitmix64(state))
        state = (state + 0x9E3779B97F4A7C15) & inputs.MASK64
    assert outs == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_frame_seeds_are_distinct_per_field():
    seeds = {inputs.frame_seed(wid, f, t) for wid in (1, 2, 3) for f in range(50) for t in "qkv"}
    assert len(seeds) == 3 * 50 * 3


def test_image_token_count_of_the_518x378_workload():
    assert math.ceil(518 / 14) * math.ceil(378 / 14) == inputs.METRIC_518x378.M == 999
    assert inputs.METRIC_518x378.Lq == 1005


def test_draw_is_deterministic_with_distinct_streams():
    w = inputs.TINY.with_(L=3)
    a = inputs.draw(w, 4, "k")
    assert a.shape == (3, w.S + w.M, w.H, w.D) and a.dtype == torch.float32
    assert torch.equal(a, inputs.draw(w, 4, "k"))
    assert not torch.equal(a, inputs.draw(w, 5, "k"))
    assert not torch.equal(a, inputs.draw(w, 4, "v"))
    assert not torch.equal(a[0], a[1])
    assert torch.equal(inputs.draw(w, 4, "k", layers=[2])[0], a[2])


def test_bf16_workload_is_the_fp32_draw_rounded():
    a = inputs.draw(inputs.TINY, 7, "q")
    b = inputs.draw(inputs.TINY_BF16, 7, "q")
    assert b.dtype == torch.bfloat16
    assert torch.equal(b, a.to(torch.bfloat16))


def test_key_norms_are_lognormal_and_shared_by_the_heads_of_a_token():
    w = inputs.WORKED_EXAMPLE.with_(dtype="f32")
    k = inputs.draw(w, 3, "k")[0].double()
    k0 = inputs.draw(w.with_(key_norm_sigma=None), 3, "k")[0].double()
    ratio = k / k0                                     # [Lq][H][D]
    per_token = ratio[:, 0, 0]
    assert torch.allclose(ratio, per_token[:, None, None].expand_as(ratio), rtol=1e-5, atol=0)
    log_s = per_token.log()
    assert abs(float(log_s.mean())) < 0.1              # 506 draws of N(0, 0.5^2)
    assert abs(float(log_s.std()) - 0.5) < 0.06
    # Q and V carry no key norms
    assert torch.equal(inputs.draw(w, 3, "v"), inputs.draw(w.with_(key_norm_sigma=None), 3, "v"))


def test_windowed_mode_windows():
    wins = inputs.WINDOWED_VO.windows()
    assert len(wins) == 179
    assert wins[0] == (0, 128) and wins[1] == (112, 128)
    assert wins[-1] == (19936, 64)
    assert sum(ln for _, ln in wins) == 20000 + 16 * 178
    assert inputs.METRIC_518x378.windows() == [(0, 10000)]
