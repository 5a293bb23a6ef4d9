"""CPU oracle for Geometric Context Attention (GCA).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s cpu_baseline leg and reference arm may import this package.  It
shares no code with the CUDA library under ``windowed_memory_attention_b200/``
and never imports it; both sides receive the same seeded inputs from
``windowed_memory_attention_b200/inputs.py``, which holds no attention
arithmetic.

Sources (LingBot-Map pages):
  * paper digest §2.2 (frame-type table): the current frame keeps all M+6
    tokens; n anchor frames keep all tokens; k pose-reference-window frames keep
    all tokens; every other earlier frame ("trajectory memory") keeps only its
    6 summary tokens;
  * paper digest §2.5 (attention-mask table): the current frame sees anchors
    (all tokens) + window frames (all tokens) + summary tokens of every history
    frame; window frames see window + anchors; trajectory-memory frames take
    part only through their summary tokens;
  * paper digest §2.4 (token-count formula): cache = M(n+k) + 6T tokens against
    (M+6)T for causal attention; the worked example M~500, n=3, k=16, T=10000
    gives about 6.95e4 against about 5.06e6 (~73x);
  * news article, mask figure caption (d): GCA with n=2 anchors, k=2 window;
  * code walkthrough §2: a frame that leaves the window drops its M image tokens
    and keeps its summary tokens; §3.2: anchors ("scale frames") form one block
    that attends within itself before single-frame streaming, and with
    keyframe_interval > 1 a non-keyframe is predicted from the cache but its
    K/V is not kept (skip-append); §3.3: the window counts keyframes entering
    the cache, not video frames.

Readings where the pages leave a step open:
  * the k-frame window counts the current frame, so after frame t the full
    frames are the anchors and t-k+1..t — the only reading under which the
    cache holds exactly M(n+k)+6T tokens once T > n+k;
  * attention inside a frame is bidirectional; causality is per frame;
  * the summary tokens of anchor and window frames are counted once;
  * in the anchor-block option the n anchors see each other's tokens in full;
  * a non-keyframe reads exactly what the latest keyframe reads as a single
    query frame, plus all of its own tokens (bidirectional).

Parity pins: tests/test_oracle_pins.py.  The one unpinned quantity is the
model's learned numbers, which this path does not compute.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from typing import Callable, Iterable, Optional, Sequence

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liboracle.so")


# ----------------------------------------------------------------------------
# closed forms (paper digest §2.4)
# ----------------------------------------------------------------------------
def cache_tokens(M: int, S: int, n: int, k: int, T: int, keep: Optional[int] = None) -> int:
    """Tokens cached by GCA after T frames: full frames hold M image tokens,
    every frame holds S summary tokens.  Full frames are the first
    min(T, n+k) frames' worth: n anchors plus the k-frame window.  With
    ``keep`` < S special tokens kept per frame (camera-only: 1; none: 0) a
    full frame holds its other S-keep special tokens with its image tokens."""
    kp = S if keep is None else keep
    return (M + S - kp) * min(T, n + k) + kp * T


def causal_tokens(M: int, S: int, T: int) -> int:
    """Tokens cached by plain causal attention after T frames: (M+S)T."""
    return (M + S) * T


# ----------------------------------------------------------------------------
# (O2) token-level visibility predicate, paper digest §2.5
# ----------------------------------------------------------------------------
def visible(i: int, j: int, tau: int, *, n: int, k: int, S: int,
            anchor_block: bool = False, keep: Optional[int] = None) -> bool:
    """May a query token of frame i attend to token slot tau of frame j?

    Slots 0..S-1 are the summary tokens (camera, anchor, 4 registers), slots
    S..S+M-1 the image tokens.  Frame i itself is part of its window.  The
    first ``keep`` slots (default all S) form the trajectory memory; the other
    special tokens are seen only while the frame is full, like image tokens.
    """
    kp = S if keep is None else keep
    if anchor_block and i < n and j < n:
        return True                       # anchors attend jointly (one block)
    if j > i:
        return False                      # no future frames
    if tau < kp:
        return True                       # kept tokens of every earlier frame
    return j < n or j >= i - k + 1        # the rest: anchors and the window


# ----------------------------------------------------------------------------
# (O1) streaming simulator: append frame, evict what left the window
# ----------------------------------------------------------------------------
def stream_state(i: int, *, n: int, k: int, anchor_block: bool = False):
    """Frames holding all tokens, and frames reduced to their summary tokens,
    in the cache that query frame i reads.

    Replays the stream: frame f enters with all tokens; then every non-anchor
    frame that is k or more frames behind f drops its image tokens (code
    walkthrough §2, compressing eviction).  With the anchor block the first n
    frames enter together, so an anchor query sees all n anchors.
    """
    full: set = set()
    summary: set = set()
    for f in range(i + 1):
        full.add(f)
        for g in sorted(full):
            if g >= n and g <= f - k:
                full.discard(g)
                summary.add(g)
    if anchor_block and i < n:
        full |= set(range(n))
    return sorted(full), sorted(summary)


FrameKV = Callable[[int, bool], "tuple[np.ndarray, np.ndarray]"]
"""frame_kv(j, summary_only) -> (K, V) of frame j for one layer, float32,
shape [S+M][H][D], or [S][H][D] when summary_only."""


def gather_keys(i: int, frame_kv: FrameKV, *, n: int, k: int, S: int,
                anchor_block: bool = False, keep: Optional[int] = None):
    """Keys and values that query frame i attends to, [Nk][H][D] float32.
    Frames reduced to their trajectory memory contribute their first ``keep``
    (default S) tokens."""
    kp = S if keep is None else keep
    full, summary = stream_state(i, n=n, k=k, anchor_block=anchor_block)
    ks, vs = [], []
    for f in full:
        kf, vf = frame_kv(f, False)
        ks.append(kf)
        vs.append(vf)
    for f in summary:
        kf, vf = frame_kv(f, True)
        ks.append(kf[:kp])
        vs.append(vf[:kp])
    return np.concatenate(ks, 0), np.concatenate(vs, 0)


# ----------------------------------------------------------------------------
# attention core: fp64 softmax attention over an explicit key set
# ----------------------------------------------------------------------------
def attention_np(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float):
    """Plain fp64 softmax attention (numpy twin of the C core).

    q [nq][H][D], k and v [nk][H][D]; returns out [nq][H][D] and natural-log
    lse [nq][H], both float64."""
    q64 = q.astype(np.float64)
    k64 = k.astype(np.float64)
    v64 = v.astype(np.float64)
    s = scale * np.einsum("rhd,uhd->hru", q64, k64)
    mx = s.max(axis=2, keepdims=True)
    p = np.exp(s - mx)
    den = p.sum(axis=2, keepdims=True)
    out = np.einsum("hru,uhd->rhd", p, v64) / den.transpose(1, 0, 2)
    lse = (mx + np.log(den))[:, :, 0].T
    return out, lse


_lib = None


def build_core(force: bool = False) -> str:
    """Compile the C core (gcc, fp64, OpenMP) next to this file."""
    src = os.path.join(HERE, "gca_oracle.c")
    if force or not os.path.exists(LIB_PATH) or \
            os.path.getmtime(LIB_PATH) < os.path.getmtime(src):
        tmp = LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, src, "-lm"])
        os.replace(tmp, LIB_PATH)
    return LIB_PATH


def _core():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build_core())
        lib.gca_oracle_attention.restype = ctypes.c_int
        lib.gca_oracle_attention.argtypes = [
            ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_double,
            ctypes.c_void_p, ctypes.c_void_p]
        lib.gca_oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def core_threads() -> int:
    return int(_core().gca_oracle_num_threads())


def attention_c(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float):
    """fp64 softmax attention through the C core; same contract as attention_np."""
    nq, H, D = q.shape
    nk = k.shape[0]
    qf = np.ascontiguousarray(q, dtype=np.float32)
    kh = np.ascontiguousarray(np.asarray(k, dtype=np.float32).transpose(1, 0, 2))
    vh = np.ascontiguousarray(np.asarray(v, dtype=np.float32).transpose(1, 0, 2))
    out = np.empty((nq, H, D), dtype=np.float64)
    lse = np.empty((nq, H), dtype=np.float64)
    rc = _core().gca_oracle_attention(
        qf.ctypes.data, nq, kh.ctypes.data, vh.ctypes.data, nk, H, D, float(scale),
        out.ctypes.data, lse.ctypes.data)
    if rc != 0:
        raise RuntimeError("oracle core failed")
    return out, lse


def attention(q, k, v, scale, impl: str = "c"):
    return attention_c(q, k, v, scale) if impl == "c" else attention_np(q, k, v, scale)


# ----------------------------------------------------------------------------
# (O1) one streaming step
# ----------------------------------------------------------------------------
def stream_step(q_block: np.ndarray, last_frame: int, frame_kv: FrameKV, *, n: int,
                k: int, S: int, scale: float, anchor_block: bool = False,
                rows: Optional[Sequence[int]] = None, impl: str = "c", keep: Optional[int] = None):
    """GCA output of the query block that ends at frame ``last_frame``.

    q_block is [F][S+M][H][D] (the F most recent frames' queries).  Returns
    out [F][R][H][D] and lse [F][R][H] in float64, where R = S+M, or
    R = len(rows) when ``rows`` picks a subset of each frame's token rows.
    """
    F = q_block.shape[0]
    outs, lses = [], []
    for b in range(F):
        i = last_frame - F + 1 + b
        kk, vv = gather_keys(i, frame_kv, n=n, k=k, S=S, anchor_block=anchor_block, keep=keep)
        qi = q_block[b] if rows is None else q_block[b][list(rows)]
        o, l = attention(qi, kk, vv, scale, impl)
        outs.append(o)
        lses.append(l)
    return np.stack(outs), np.stack(lses)


# ----------------------------------------------------------------------------
# non-keyframe steps (code walkthrough §3.2: keyframe_interval; paper digest
# §5.1: not every frame enters the memory)
# ----------------------------------------------------------------------------
def is_keyframe(x: int, *, n: int, interval: int) -> bool:
    """Does video frame x enter the cache?  The first n (scale) frames always
    do; after them every interval-th frame, counting from frame n, does."""
    return x < n or interval <= 1 or (x - n) % interval == 0


def latest_keyframe(x: int, *, n: int, interval: int) -> int:
    """Cache index of the latest keyframe among video frames 0..x (the cache
    numbers keyframes 0, 1, 2, ... in the order they enter); -1 if none."""
    return sum(1 for y in range(x + 1) if is_keyframe(y, n=n, interval=interval)) - 1


def transient_step(q: np.ndarray, own_k: np.ndarray, own_v: np.ndarray, last_key: int,
                   frame_kv: FrameKV, *, n: int, k: int, S: int, scale: float,
                   anchor_block: bool = False, rows: Optional[Sequence[int]] = None,
                   impl: str = "c", keep: Optional[int] = None):
    """Output of a non-keyframe, q / own_k / own_v [S+M][H][D].

    The frame is predicted like every other frame but its K/V never enters the
    cache: its queries read what the latest keyframe (cache index last_key)
    reads as a single query frame, plus all of its own tokens.  With no
    keyframe yet (last_key < 0) they read only their own tokens.  Returns out
    [R][H][D] and lse [R][H] in float64.
    """
    ks, vs = [], []
    if last_key >= 0:
        kk, vv = gather_keys(last_key, frame_kv, n=n, k=k, S=S, anchor_block=anchor_block,
                             keep=keep)
        ks.append(kk)
        vs.append(vv)
    ks.append(own_k)
    vs.append(own_v)
    qi = q if rows is None else q[list(rows)]
    return attention(qi, np.concatenate(ks, 0), np.concatenate(vs, 0), scale, impl)


def bruteforce_keyframes(Q: np.ndarray, K: np.ndarray, V: np.ndarray, *, n: int, k: int,
                         S: int, interval: int, scale: float, anchor_block: bool = False,
                         keep: Optional[int] = None):
    """Every video frame's output at once for a stream in which only keyframes
    are cached.  Q, K, V [X][S+M][H][D] over all X video frames.  A query of
    frame x sees token tau of keyframe y when the token rule allows it between
    the cache indices of x's latest keyframe and of y, and, when x itself is
    not a keyframe, every token of x.  Returns out [X][S+M][H][D], lse
    [X][S+M][H] (float64)."""
    X, Lq, H, D = Q.shape
    kid = {}
    for y in range(X):
        if is_keyframe(y, n=n, interval=interval):
            kid[y] = len(kid)
    q = Q.astype(np.float64)
    kf = K.reshape(X * Lq, H, D).astype(np.float64)
    vf = V.reshape(X * Lq, H, D).astype(np.float64)
    outs, lses = [], []
    for x in range(X):
        i = latest_keyframe(x, n=n, interval=interval)
        vis = np.zeros(X * Lq, dtype=bool)
        for y in range(X):
            for tau in range(Lq):
                if y in kid and i >= 0:
                    vis[y * Lq + tau] = visible(i, kid[y], tau, n=n, k=k, S=S,
                                                anchor_block=anchor_block, keep=keep)
                if y == x and x not in kid:
                    vis[y * Lq + tau] = True
        o, l = attention_np(q[x], kf[vis], vf[vis], scale)
        outs.append(o)
        lses.append(l)
    return np.stack(outs), np.stack(lses)


# ----------------------------------------------------------------------------
# (O2) brute force over the whole sequence with an explicit mask
# ----------------------------------------------------------------------------
def visibility_mask(T: int, Lq: int, *, n: int, k: int, S: int,
                    anchor_block: bool = False, keep: Optional[int] = None) -> np.ndarray:
    """Boolean [T*Lq][T*Lq] mask of the whole stream from the token rule."""
    keys = [(j, tau) for j in range(T) for tau in range(Lq)]
    frame_rows = np.zeros((T, T * Lq), dtype=bool)
    for i in range(T):
        for b, (j, tau) in enumerate(keys):
            frame_rows[i, b] = visible(i, j, tau, n=n, k=k, S=S, anchor_block=anchor_block,
                                       keep=keep)
    return np.repeat(frame_rows, Lq, axis=0)


def bruteforce(Q: np.ndarray, K: np.ndarray, V: np.ndarray, *, n: int, k: int, S: int,
               scale: float, anchor_block: bool = False, keep: Optional[int] = None):
    """Every frame's GCA output at once: Q, K, V [T][S+M][H][D] -> out
    [T][S+M][H][D], lse [T][S+M][H] (float64)."""
    T, Lq, H, D = Q.shape
    q = Q.reshape(T * Lq, H, D).astype(np.float64)
    kx = K.reshape(T * Lq, H, D).astype(np.float64)
    vx = V.reshape(T * Lq, H, D).astype(np.float64)
    mask = visibility_mask(T, Lq, n=n, k=k, S=S, anchor_block=anchor_block, keep=keep)
    s = scale * np.einsum("rhd,uhd->hru", q, kx)
    s = np.where(mask[None], s, -np.inf)
    mx = s.max(axis=2, keepdims=True)
    p = np.exp(s - mx)
    den = p.sum(axis=2, keepdims=True)
    out = np.einsum("hru,uhd->rhd", p, vx) / den.transpose(1, 0, 2)
    lse = (mx + np.log(den))[:, :, 0].T
    return out.reshape(T, Lq, H, D), lse.reshape(T, Lq, H)


def frame_visibility_matrix(T: int, *, n: int, k: int, S: int, anchor_block: bool = False):
    """Frame-level picture of the mask: entry [i][j] is 'F' (all tokens of frame
    j visible to frame i), 'S' (summary tokens only) or '.' (none)."""
    M_probe = 1
    rows = []
    for i in range(T):
        row = []
        for j in range(T):
            summ = visible(i, j, 0, n=n, k=k, S=S, anchor_block=anchor_block)
            img = visible(i, j, S + M_probe - 1, n=n, k=k, S=S, anchor_block=anchor_block)
            row.append("F" if img and summ else ("S" if summ else "."))
        rows.append("".join(row))
    return rows


# ----------------------------------------------------------------------------
# 3D rotary position encoding (video RoPE) on Q and K
# ----------------------------------------------------------------------------
# Sources: the news article's ablation (context tokens together with video RoPE
# raise AUC@3), paper digest §2.7 (a temporal positional encoding PE(t) on the
# trajectory memory's summary tokens, taken from the WAN video model), the code
# walkthrough §3.1 (enable_3d_rope is a first-class constructor flag) and the
# paper-to-code article §3 (3D RoPE carries the position along the time axis).
# The formula is not printed; the reading taken here is rotary position
# encoding (Su et al., "RoFormer", 2021) over three axes, time t, patch row y
# and patch column x:
#   * the D=64 head dims are split into three contiguous parts, 24 dims for t,
#     20 for y, 20 for x (time takes the larger share);
#   * inside a part of d dims, dims (2i, 2i+1) form pair i, rotated by the angle
#     pos * base^(-2i/d) with base 10000: (a, b) -> (a cos - b sin, a sin + b cos);
#   * image token m of frame t (row-major over a grid_w-wide patch grid) sits at
#     (t, m // grid_w, m % grid_w); the frame's special tokens at (t, 0, 0), so
#     they carry only the timestamp;
#   * t is the frame's index in the cache (frames since create or reset);
#   * Q and K are rotated, V is not; the rotated vectors are held in the
#     workload's dtype, as a model running in that dtype holds them.
ROPE_SPLIT = (24, 20, 20)
ROPE_BASE = 10000.0


def rope_angles(t: float, y: float, x: float, D: int = 64, base: float = ROPE_BASE,
                split=ROPE_SPLIT) -> np.ndarray:
    """Rotation angle of each of the D/2 dim pairs at position (t, y, x)."""
    assert sum(split) == D and all(d % 2 == 0 for d in split)
    out = []
    for pos, d in zip((t, y, x), split):
        i = np.arange(d // 2, dtype=np.float64)
        out.append(pos * base ** (-2.0 * i / d))
    return np.concatenate(out)


def rope_matrix(t: float, y: float, x: float, D: int = 64, base: float = ROPE_BASE,
                split=ROPE_SPLIT) -> np.ndarray:
    """The explicit [D][D] rotation: block diagonal, one 2x2 rotation per pair."""
    R = np.zeros((D, D), dtype=np.float64)
    for i, a in enumerate(rope_angles(t, y, x, D, base, split)):
        c, s = math.cos(a), math.sin(a)
        R[2 * i, 2 * i], R[2 * i, 2 * i + 1] = c, -s
        R[2 * i + 1, 2 * i], R[2 * i + 1, 2 * i + 1] = s, c
    return R


def token_positions(frame: int, S: int, M: int, grid_w: int):
    """(t, y, x) of the S + M tokens of a frame (special tokens first)."""
    pos = [(frame, 0, 0)] * S
    pos += [(frame, m // grid_w, m % grid_w) for m in range(M)]
    return pos


def round_to_dtype(x: np.ndarray, dtype: str) -> np.ndarray:
    """Values as held in `dtype` ("f32" or "bf16", round to nearest even),
    returned as float64.  bf16 keeps the top 16 bits of the float32 pattern."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    if dtype == "f32":
        return f.astype(np.float64)
    b = f.view(np.uint32).astype(np.uint64)
    b = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) & np.uint64(0xFFFF0000)
    return b.astype(np.uint32).view(np.float32).astype(np.float64)


def rope_frame(x: np.ndarray, frame: int, *, S: int, grid_w: int, dtype: str,
               base: float = ROPE_BASE) -> np.ndarray:
    """Rotate every token of one frame, x [S+M][H][D], by its position's
    explicit rotation matrix (the same for every head), then hold the result
    in `dtype`.  Returns float32."""
    Lq, H, D = x.shape
    out = np.empty((Lq, H, D), dtype=np.float64)
    cache = {}
    for u, p in enumerate(token_positions(frame, S, Lq - S, grid_w)):
        R = cache.get(p)
        if R is None:
            R = cache[p] = rope_matrix(*p, D=D, base=base)
        out[u] = x[u].astype(np.float64) @ R.T
    return round_to_dtype(out, dtype).astype(np.float32)
