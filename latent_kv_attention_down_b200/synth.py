"""Seeded synthetic inputs for the latent-KV chunk attention path.

This module only draws numbers: Gaussian activations, queries and weights
with the shapes of a Wan2.1-T2V-1.3B attention layer (or a tiny stand-in),
rounded to bf16 where the workload stores bf16.  It holds none of the
method's arithmetic, so both the fp64 oracle (through the tests) and the CUDA
path (through the tests and the benchmark) consume the same values.

Recipe
------
* every tensor is drawn from its own PCG64 stream, seeded by
  ``SeedSequence([base_seed, workload_id, layer, chunk, pass, tensor_id])``;
* activations ``x ~ N(0, 1)``, queries ``q ~ N(0, 1)``;
* weights ``W ~ N(0, 1/fan_in)``: ``W_down`` has fan-in ``d_model``,
  ``W_uk`` and ``W_uv`` have fan-in ``d_latent``;
* bf16 workloads round every value to bf16 (round to nearest even) and keep
  it in a float32 array, so the same bits can be handed to either side.
"""
from __future__ import annotations

import dataclasses
import hashlib

import numpy as np

# tensor ids inside a seed sequence
_T_X, _T_Q, _T_WDOWN, _T_WUK, _T_WUV = 1, 2, 3, 4, 5
_T_WO, _T_CQ, _T_WUQ, _T_WQR = 9, 10, 11, 12


@dataclasses.dataclass(frozen=True)
class Dims:
    """Shape of one latent attention layer and of its sliding window."""

    name: str
    d_model: int
    n_heads: int
    d_nope: int
    d_rope: int
    d_latent: int
    rope_pairs: tuple  # complex pairs for the (t, h, w) axes
    grid_h: int
    grid_w: int
    window_frames: int  # ring capacity in frames, current chunk included
    chunk_frames: int
    batch: int = 1
    dtype: str = "bf16"  # storage type of every tensor: "bf16" or "fp32"
    rope_theta: float = 10000.0
    rope_base_dims: tuple = (0, 0, 0)  # 0 = twice the pair count of the axis
    sink_frames: int = 0  # leading frames pinned in the ring (window_frames counts them)
    d_q: int = 768  # query latent width

    @property
    def d_head(self) -> int:
        return self.d_nope + self.d_rope

    @property
    def tokens_per_frame(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def n_queries(self) -> int:
        return self.chunk_frames * self.tokens_per_frame

    @property
    def window_tokens(self) -> int:
        return self.window_frames * self.tokens_per_frame

    def replace(self, **kw) -> "Dims":
        return dataclasses.replace(self, **kw)


# The tiny fp32 case: two heads of 16 dims (10 content + 6 positional, one
# complex pair per axis), latent of 8, a 4x6 frame grid, a window of 4 frames
# of which the newest one is the current chunk.
TINY = Dims("tiny", d_model=32, n_heads=2, d_nope=10, d_rope=6, d_latent=8,
            rope_pairs=(1, 1, 1), grid_h=4, grid_w=6, window_frames=4,
            chunk_frames=1, dtype="fp32")

# One Wan2.1-T2V-1.3B-shaped layer: model dim 1536, 12 heads of 128
# (96 content + 32 positional in (6, 5, 5) pairs), latent 192, a 30x52
# latent grid, chunks of 3 latent frames, a 21-frame window.
WAN = Dims("wan", d_model=1536, n_heads=12, d_nope=96, d_rope=32, d_latent=192,
           rope_pairs=(6, 5, 5), grid_h=30, grid_w=52, window_frames=21,
           chunk_frames=3)

# The same layer on a 10x20 grid: small enough for the full fp64 oracle in a
# second, large enough for several query and key tiles with ragged tails.
WAN_SMALL = WAN.replace(name="wan_small", grid_h=10, grid_w=20)

# Long-horizon inference as the pages run it: one sink latent frame and the six most recent latent
# frames (the current chunk among them), 7 x 1560 = 10920 keys.
WAN_SINK = WAN.replace(name="wan_sink", window_frames=7, sink_frames=1)
WAN_SMALL_SINK = WAN_SMALL.replace(name="wan_small_sink", window_frames=7, sink_frames=1)

WORKLOADS = {d.name: d for d in (TINY, WAN, WAN_SMALL, WAN_SINK, WAN_SMALL_SINK)}


def _workload_id(name: str) -> int:
    return int.from_bytes(hashlib.blake2b(name.encode(), digest_size=4).digest(), "little")


def rng(dims: Dims, layer: int, chunk: int, pass_: int, tensor: int,
        base_seed: int = 0) -> np.random.Generator:
    ss = np.random.SeedSequence([base_seed, _workload_id(dims.name), layer, chunk, pass_, tensor])
    return np.random.Generator(np.random.PCG64(ss))


def bf16_round(a) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); float32 out."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def _store(dims: Dims, a: np.ndarray) -> np.ndarray:
    a = a.astype(np.float32)
    return bf16_round(a) if dims.dtype == "bf16" else a


def gaussian(dims: Dims, shape, std: float, layer: int, chunk: int, pass_: int,
             tensor: int, base_seed: int = 0) -> np.ndarray:
    g = rng(dims, layer, chunk, pass_, tensor, base_seed)
    return _store(dims, g.standard_normal(shape, dtype=np.float32) * np.float32(std))


@dataclasses.dataclass
class LayerWeights:
    w_down: np.ndarray  # [d_latent + d_rope, d_model]: rows 0..d_latent-1 are W_dkv, the rest W_kr
    w_uk: np.ndarray    # [n_heads, d_nope, d_latent]
    w_uv: np.ndarray    # [n_heads, d_head, d_latent]
    w_o: np.ndarray = None  # [d_model, n_heads * d_head], the output mixer


def weights(dims: Dims, layer: int = 0, base_seed: int = 0) -> LayerWeights:
    d = dims
    w_down = gaussian(d, (d.d_latent + d.d_rope, d.d_model), d.d_model ** -0.5, layer, 0, 0, _T_WDOWN, base_seed)
    w_uk = gaussian(d, (d.n_heads, d.d_nope, d.d_latent), d.d_latent ** -0.5, layer, 0, 0, _T_WUK, base_seed)
    w_uv = gaussian(d, (d.n_heads, d.d_head, d.d_latent), d.d_latent ** -0.5, layer, 0, 0, _T_WUV, base_seed)
    w_o = gaussian(d, (d.d_model, d.n_heads * d.d_head), (d.n_heads * d.d_head) ** -0.5, layer, 0, 0, _T_WO,
                   base_seed)
    return LayerWeights(w_down, w_uk, w_uv, w_o)


def query_latent_weights(dims: Dims, layer: int = 0, base_seed: int = 0):
    """W_uq [n_heads, d_nope, d_q] and W_qr [n_heads, d_rope, d_q], N(0, 1/d_q)."""
    d = dims
    w_uq = gaussian(d, (d.n_heads, d.d_nope, d.d_q), d.d_q ** -0.5, layer, 0, 0, _T_WUQ, base_seed)
    w_qr = gaussian(d, (d.n_heads, d.d_rope, d.d_q), d.d_q ** -0.5, layer, 0, 0, _T_WQR, base_seed)
    return w_uq, w_qr


def query_latents(dims: Dims, layer: int, chunk: int, pass_: int = 0, base_seed: int = 0) -> np.ndarray:
    """c_Q of one chunk: [batch, chunk_frames * tokens_per_frame, d_q], N(0, 1)."""
    return gaussian(dims, (dims.batch, dims.n_queries, dims.d_q), 1.0, layer, chunk, pass_, _T_CQ, base_seed)


def activations(dims: Dims, layer: int, chunk: int, pass_: int = 0, n_frames: int | None = None,
                base_seed: int = 0) -> np.ndarray:
    """x for one appended chunk: [batch, n_frames * tokens_per_frame, d_model]."""
    nf = dims.chunk_frames if n_frames is None else n_frames
    return gaussian(dims, (dims.batch, nf * dims.tokens_per_frame, dims.d_model), 1.0,
                    layer, chunk, pass_, _T_X, base_seed)


def queries(dims: Dims, layer: int, chunk: int, pass_: int = 0, n_frames: int | None = None,
            std: float = 1.0, base_seed: int = 0) -> np.ndarray:
    """Per-head queries for one chunk: [batch, n_frames * tokens_per_frame, n_heads, d_head],
    each head laid out as [content (d_nope) | positional (d_rope)]."""
    nf = dims.chunk_frames if n_frames is None else n_frames
    return gaussian(dims, (dims.batch, nf * dims.tokens_per_frame, dims.n_heads, dims.d_head), std,
                    layer, chunk, pass_, _T_Q, base_seed)


# ---------------------------------------------------------------- long rollouts
_T_XPOOL, _T_QPOOL, _T_PICK = 6, 7, 8


class FramePool:
    """Inputs for rollouts of thousands of calls (30 layers x 20 chunks x 4
    passes at the Wan-1.3B layer shape) without drawing 7 M fresh normals per
    call: a pool of ``n_pool`` seeded Gaussian frames of activations and of
    queries is drawn once; frame k of a call is pool entry e, its token rows
    cyclically shifted by s and its sign flipped by g, with (e, s, g) drawn from
    the call's own seeded stream.  The values stay N(0, 1) (bf16 where the
    workload is bf16), every call still sees different content at every token,
    and the pick is exact on either a NumPy array or a torch tensor, so the
    oracle and the CUDA path get the same bits."""

    def __init__(self, dims: Dims, n_pool: int = 8, base_seed: int = 0):
        self.dims = dims
        self.base_seed = base_seed
        T = dims.tokens_per_frame
        self.x = gaussian(dims, (n_pool, T, dims.d_model), 1.0, 0, 0, 0, _T_XPOOL, base_seed)
        self.q = gaussian(dims, (n_pool, T, dims.n_heads, dims.d_head), 1.0, 0, 0, 0, _T_QPOOL, base_seed)

    def picks(self, layer: int, chunk: int, pass_: int, tensor: int):
        """[(entry, shift, sign)] for every (sample, frame) of the call, sample-major."""
        d = self.dims
        g = rng(d, layer, chunk, pass_, _T_PICK * 16 + tensor, self.base_seed)
        n = d.batch * d.chunk_frames
        e = g.integers(0, self.x.shape[0], n)
        s = g.integers(0, d.tokens_per_frame, n)
        sg = np.where(g.integers(0, 2, n) == 1, -1.0, 1.0)
        return list(zip(e.tolist(), s.tolist(), sg.tolist()))

    @staticmethod
    def _take(pool, picks, batch):
        if isinstance(pool, np.ndarray):
            frames = [np.roll(pool[e], s, axis=0) * np.float32(g) for e, s, g in picks]
            out = np.concatenate(frames, axis=0)
        else:
            import torch
            frames = [torch.roll(pool[e], s, dims=0) * g for e, s, g in picks]
            out = torch.cat(frames, dim=0)
        return out.reshape((batch, -1) + tuple(out.shape[1:]))

    def activations(self, layer: int, chunk: int, pass_: int = 0, pool=None):
        """x of one chunk [batch, chunk_frames * T, d_model]; ``pool`` may be a
        device copy of ``self.x`` (same values) to build it on the device."""
        return self._take(self.x if pool is None else pool, self.picks(layer, chunk, pass_, _T_X), self.dims.batch)

    def queries(self, layer: int, chunk: int, pass_: int = 0, pool=None):
        """q of one chunk [batch, chunk_frames * T, n_heads, d_head]."""
        return self._take(self.q if pool is None else pool, self.picks(layer, chunk, pass_, _T_Q), self.dims.batch)
