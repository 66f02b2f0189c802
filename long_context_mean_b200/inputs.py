"""Seeded synthetic inputs and the five workload descriptions.

This module draws random numbers and shapes them into Q, K, V; it holds none
of the attention method's arithmetic, and both the CUDA path's tests/bench
and the CPU oracle take their inputs from it.  Every tensor is generated on
the host with NumPy's PCG64, per (tensor, batch, head) from its own seed
sequence, so any head can be regenerated alone; values are rounded to bf16
(round to nearest even) and returned both as raw bf16 bit patterns
(uint16) and as the exactly widened float32.

Token order is raster frame-major over the latent (i = t*H*W + h*W + w)
with text tokens appended, the order of the pages' video examples.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import numpy as np


# ----------------------------------------------------------------------------
# bf16 rounding
# ----------------------------------------------------------------------------

def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit pattern, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def round_bf16(x: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(to_bf16_bits(x))


# ----------------------------------------------------------------------------
# Workload descriptions
# ----------------------------------------------------------------------------

@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    B: int
    Hq: int
    Hkv: int
    T: int
    H: int
    W: int
    txt_len: int
    d: int
    dv: int
    dtype: str                      # "bf16" or "fp32"
    generator: str                  # "iid", "field", "lowrank"
    order: str = "identity"         # "identity", "window", "hilbert"
    win: tuple = (1, 1, 1)
    sink_frames: int = 0
    bq: int = 128
    bk: int = 64
    tau: float = 0.9
    theta: float = 0.0
    lam: float = -math.inf
    causal: bool = False
    local_window: int = 0
    anchor_tokens: int = 0
    sigma: tuple = (0.0, 4.0, 4.0)  # blur sigma along (t, h, w) in tokens
    shift: tuple = (0, 0)           # content shift per frame along (h, w)
    noise: float = 0.3
    rank: int = 16
    sigma_pos: float = 256.0
    target_sparsity: float = 0.0
    extra: dict = field(default_factory=dict)

    @property
    def N(self) -> int:
        return self.T * self.H * self.W + self.txt_len

    @property
    def frame_tokens(self) -> int:
        return self.H * self.W

    @property
    def sink_tokens(self) -> int:
        return self.sink_frames * self.frame_tokens

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# tau values marked "tuned" were bisected on the oracle's mask to the target
# block sparsity by oracle/tune_tau.py and frozen here.
WORKLOADS = {
    # Toy ledger of the worked example: 4 frames of 4x4, d = dv = 16, fp32.
    "toy": Workload("toy", 7, 1, 1, 1, 4, 4, 4, 0, 16, 16, "fp32", "iid",
                    bq=16, bk=16, tau=0.9, theta=0.5),
    # Image DiT attention, [1,64,64] grid.
    "image": Workload("image", 1002, 2, 24, 24, 1, 64, 64, 0, 128, 128, "bf16", "field",
                      bq=128, bk=64, tau=0.5, theta=0.6, sigma=(0.0, 4.0, 4.0),
                      target_sparsity=0.6),
    # Video DiT attention, [13,30,52] + 226 text tokens, [2,8,8] windows; the
    # similarity guard is not part of this workload's recipe (off); tau tuned
    # to block sparsity 0.80 (oracle: 0.8002).
    "video": Workload("video", 1003, 1, 24, 24, 13, 30, 52, 226, 128, 128, "bf16", "field",
                      order="window", win=(2, 8, 8), sink_frames=1, bq=128, bk=64,
                      tau=0.375, theta=0.0, lam=-5.0, sigma=(1.5, 3.0, 3.0), shift=(0, 2),
                      target_sparsity=0.8),
    # Large video attention, [21,45,80], Hilbert curve.
    "video_large": Workload("video_large", 1004, 1, 24, 24, 21, 45, 80, 0, 128, 128, "bf16",
                            "field", order="hilbert", sink_frames=1, bq=128, bk=64,
                            tau=0.5, theta=0.6, lam=-5.0, sigma=(1.5, 3.0, 3.0),
                            shift=(3, 3), target_sparsity=0.85),
    # The image and large-video workloads at the block sparsity their recipes
    # name (0.6, 0.85).  Under theta = 0.6 the smooth-field blocks (mean
    # cosine about 0.5) force every block, so the guard is off here, as for
    # the video workload; tau tuned (oracle: 0.6042 and 0.8513).
    "image_s60": Workload("image_s60", 1002, 2, 24, 24, 1, 64, 64, 0, 128, 128, "bf16", "field",
                          bq=128, bk=64, tau=0.78125, theta=0.0, sigma=(0.0, 4.0, 4.0),
                          target_sparsity=0.6),
    "video_large_s85": Workload("video_large_s85", 1004, 1, 24, 24, 21, 45, 80, 0, 128, 128, "bf16",
                                "field", order="hilbert", sink_frames=1, bq=128, bk=64,
                                tau=0.25, theta=0.0, lam=-5.0, sigma=(1.5, 3.0, 3.0),
                                shift=(3, 3), target_sparsity=0.85),
    # Causal long-context LM attention, GQA 32/8, 128K tokens.
    "lm_causal": Workload("lm_causal", 1005, 1, 32, 8, 1, 1, 131072, 0, 128, 128, "bf16",
                          "lowrank", bq=128, bk=64, tau=0.95, theta=0.0, causal=True,
                          local_window=4096, anchor_tokens=128),
}


# ----------------------------------------------------------------------------
# Generators
# ----------------------------------------------------------------------------

_TENSOR_ID = {"q": 1, "k": 2, "v": 3, "field": 4, "z": 5, "a": 6}


def _rng(seed: int, tensor: str, b: int, h: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([seed, _TENSOR_ID[tensor], b, h]))


def _gauss_kernel_fft(n: int, sigma: float) -> np.ndarray:
    """Frequency response of a circular Gaussian blur of width sigma tokens."""
    if sigma <= 0 or n == 1:
        return np.ones(n)
    f = np.fft.fftfreq(n)
    return np.exp(-2.0 * (math.pi * sigma * f) ** 2)


def _smooth_field(w: Workload, b: int, h: int) -> np.ndarray:
    """White noise over [d, T, H, W] blurred by a separable circular Gaussian,
    each channel normalised to zero mean and unit std, content shifted by
    ``shift`` tokens per frame (motion).  Returns [T*H*W, d] float64."""
    g = _rng(w.seed, "field", b, h).standard_normal((w.d, w.T, w.H, w.W))
    spec = np.fft.fftn(g, axes=(1, 2, 3))
    kt = _gauss_kernel_fft(w.T, w.sigma[0])[:, None, None]
    kh = _gauss_kernel_fft(w.H, w.sigma[1])[None, :, None]
    kw = _gauss_kernel_fft(w.W, w.sigma[2])[None, None, :]
    f = np.real(np.fft.ifftn(spec * (kt * kh * kw)[None], axes=(1, 2, 3)))
    f -= f.mean(axis=(1, 2, 3), keepdims=True)
    f /= f.std(axis=(1, 2, 3), keepdims=True)
    if w.shift != (0, 0):
        for t in range(w.T):
            f[:, t] = np.roll(f[:, t], (w.shift[0] * t, w.shift[1] * t), axis=(1, 2))
    return f.reshape(w.d, -1).T


def _lowrank_basis(w: Workload, b: int) -> np.ndarray:
    """Z in R^{N x rank}: white noise blurred along the sequence (circular
    Gaussian, sigma_pos tokens), unit std per component."""
    z = _rng(w.seed, "z", b, 0).standard_normal((w.N, w.rank))
    k = _gauss_kernel_fft(w.N, w.sigma_pos)[:, None]
    z = np.real(np.fft.ifft(np.fft.fft(z, axis=0) * k, axis=0))
    z -= z.mean(axis=0, keepdims=True)
    z /= z.std(axis=0, keepdims=True)
    return z


def gen_head(w: Workload, tensor: str, b: int, h: int, _cache=None) -> np.ndarray:
    """One head of Q, K or V as float32 [N, d] (before bf16 rounding).

    h is a query head for "q" and a kv head for "k"/"v"."""
    n_video = w.T * w.H * w.W
    dim = w.dv if tensor == "v" else w.d
    if w.generator == "iid" or tensor == "v":
        return _rng(w.seed, tensor, b, h).standard_normal((w.N, dim)).astype(np.float32)
    if w.generator == "field":
        out = np.empty((w.N, dim), dtype=np.float64)
        kv_head = h if tensor == "k" else h * w.Hkv // w.Hq
        fld = _smooth_field(w, b, kv_head) if _cache is None else _cache
        eps = _rng(w.seed, tensor, b, h).standard_normal((w.N, dim))
        out[:n_video] = fld + w.noise * eps[:n_video]
        out[n_video:] = eps[n_video:]
        return out.astype(np.float32)
    if w.generator == "lowrank":
        z = _lowrank_basis(w, b) if _cache is None else _cache
        g = h if tensor == "k" else h // (w.Hq // w.Hkv)
        a = _rng(w.seed, "a", b, g).standard_normal((w.rank, dim)) / math.sqrt(w.rank)
        eps = _rng(w.seed, tensor, b, h).standard_normal((w.N, dim))
        return (z @ a + eps).astype(np.float32)
    raise ValueError(w.generator)


def gen_qkv(w: Workload, heads=None, batches=None):
    """Q, K, V for a workload as dict of float32 arrays (bf16-rounded when
    the workload is bf16) plus the raw bf16 bit patterns.

    ``heads``/``batches`` restrict generation to a subset of query heads
    (K/V then hold the kv heads those query heads read, in order); by
    default everything is generated: q [B, Hq, N, d], k/v [B, Hkv, N, d].
    """
    batches = list(range(w.B)) if batches is None else list(batches)
    qheads = list(range(w.Hq)) if heads is None else list(heads)
    group = w.Hq // w.Hkv
    kvheads = sorted({h // group for h in qheads}) if heads is not None else list(range(w.Hkv))
    q = np.empty((len(batches), len(qheads), w.N, w.d), dtype=np.float32)
    k = np.empty((len(batches), len(kvheads), w.N, w.d), dtype=np.float32)
    v = np.empty((len(batches), len(kvheads), w.N, w.dv), dtype=np.float32)
    for bi, b in enumerate(batches):
        shared = _lowrank_basis(w, b) if w.generator == "lowrank" else None
        fields = {}
        for gi, g in enumerate(kvheads):
            if w.generator == "field":
                fields[g] = _smooth_field(w, b, g)
            k[bi, gi] = gen_head(w, "k", b, g, fields.get(g, shared))
            v[bi, gi] = gen_head(w, "v", b, g)
        for hi, h in enumerate(qheads):
            g = h // group
            if w.generator == "field" and g not in fields:
                fields[g] = _smooth_field(w, b, g)
            q[bi, hi] = gen_head(w, "q", b, h, fields.get(g, shared))
    out = {"q": q, "k": k, "v": v, "heads": qheads, "kv_heads": kvheads, "batches": batches}
    if w.dtype == "bf16":
        for name in ("q", "k", "v"):
            bits = to_bf16_bits(out[name])
            out[name + "_bits"] = bits
            out[name] = bf16_bits_to_f32(bits)
    return out


# ----------------------------------------------------------------------------
# The worked example and the counterexample of the error-and-layout page
# ----------------------------------------------------------------------------

def worked_example_inputs():
    """The two synthetic heads of the worked example: a 4x4x4 grid, q = k
    with a one-hot of amplitude 6 on the frame dimension (head 0) or on the
    position dimension (head 1), N(0, 0.15^2) noise, values N(0, 1) of width
    3; default_rng(7) drawn noise first, values second (float64)."""
    rng = np.random.default_rng(7)
    T = H = W = 4
    P = H * W
    n, d = T * P, T + P
    frame = np.repeat(np.arange(T), P)
    pixel = np.tile(np.arange(P), T)
    q = np.zeros((2, n, d))
    q[0, np.arange(n), frame] = 6.0
    q[1, np.arange(n), T + pixel] = 6.0
    q += rng.normal(0.0, 0.15, size=q.shape)
    v = rng.normal(size=(n, 3))
    return {"q": q, "k": q.copy(), "v": v, "frame": frame, "pixel": pixel, "T": T, "P": P}


def biased_video_heads(T, H, W, txt_len, bias, d=128, dv=128, seed=0, amp=15.0, noise=0.15):
    """Heads biased to one frame or to one position, the worked example's
    construction carried to any grid and head width: head h gets
    q = k = amp * code[g(i)] + N(0, noise^2) on video token i, where g is the
    frame ("frame" bias) or the position ("position" bias) of the token and
    the codes are random unit vectors of R^d (one per frame or position);
    text tokens get noise only; v ~ N(0, 1).  bias: one "frame"/"position"
    per head.  Returns float32 [1, heads, N, d|dv] arrays, bf16-rounded, and
    their bit patterns (q_bits, k_bits, v_bits)."""
    P = H * W
    nv = T * P
    n = nv + txt_len
    frame = np.repeat(np.arange(T), P)
    pixel = np.tile(np.arange(P), T)
    q = np.empty((1, len(bias), n, d), dtype=np.float32)
    v = np.empty((1, len(bias), n, dv), dtype=np.float32)
    for h, kind in enumerate(bias):
        rng = np.random.default_rng(np.random.SeedSequence([seed, 7919, h]))
        groups = T if kind == "frame" else P
        codes = rng.standard_normal((groups, d))
        codes /= np.linalg.norm(codes, axis=1, keepdims=True)
        x = noise * rng.standard_normal((n, d))
        x[:nv] += amp * codes[frame if kind == "frame" else pixel]
        q[0, h] = x
        v[0, h] = rng.standard_normal((n, dv))
    out = {}
    for name, arr in (("q", q), ("k", q.copy()), ("v", v)):
        bits = to_bf16_bits(arr)
        out[name + "_bits"] = bits
        out[name] = bf16_bits_to_f32(bits)
    return out


def two_key_inputs():
    """q = [1], keys [ln 99, 0], values [0, 100]: probabilities 0.99 / 0.01."""
    return {"q": np.array([[1.0]]), "k": np.array([[math.log(99.0)], [0.0]]),
            "v": np.array([[0.0], [100.0]])}
