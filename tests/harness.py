"""Rollouts through libvmla next to the fp64 oracle on the same seeded inputs.

Test infrastructure: used by the GPU tests and by ``__graft_entry__.smoke()``.
"""
from __future__ import annotations

import numpy as np

import oracle.vmla_oracle as O
from latent_kv_attention_down_b200 import api, synth


def torch_dtype(dims):
    import torch
    return torch.bfloat16 if dims.dtype == "bf16" else torch.float32


def to_dev(a, dims):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).to(device="cuda", dtype=torch_dtype(dims)).contiguous()


def rel_l2(got, ref):
    return float(np.linalg.norm((got - ref).ravel()) / max(np.linalg.norm(ref.ravel()), 1e-300))


def assert_bf16_close(got, ref, what="", max_abs=3e-2):
    """The bf16 gate: relative L2 <= 1e-2 and max |err| <= 3e-2 * RMS(ref).  A caller
    may widen the max-abs term (never the relative L2 one) where the rounding of
    the design itself is shown to exceed it; it says why next to the call."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    rel = rel_l2(got, ref)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    mx = float(np.max(np.abs(got - ref)))
    assert rel <= 1e-2, f"{what}: relative L2 {rel:.3e} > 1e-2"
    assert mx <= max_abs * rms, f"{what}: max abs err {mx:.3e} > {max_abs:g} * rms {rms:.3e}"
    return rel, mx / rms


def assert_fp32_close(got, ref, what=""):
    rel = rel_l2(np.asarray(got, np.float64), np.asarray(ref, np.float64))
    assert rel <= 1e-5, f"{what}: relative L2 {rel:.3e} > 1e-5"
    return rel


class Rollout:
    """Chunks of seeded frames appended to the library's ring, remembered per
    sample so the oracle can rebuild the window from x."""

    def __init__(self, dims, layers=1, rope_mode=api.ROPE_AT_READ, design=api.DESIGN_AUTO, dense=False,
                 base_seed=0, rescale_log2=8.0):
        self.dims = dims
        self.rope_mode = rope_mode
        self.cfg = api.config_from_dims(dims, layers, rope_mode)
        self.cfg.softmax_rescale_log2 = rescale_log2
        self.m = api.LatentKVAttention(self.cfg).allocate(design=design, dense=dense)
        self.base_seed = base_seed
        self.w = [synth.weights(dims, l, base_seed) for l in range(layers)]
        self.wd = [(to_dev(w.w_down, dims), to_dev(w.w_uk, dims), to_dev(w.w_uv, dims)) for w in self.w]
        self.frame_x = [[{} for _ in range(dims.batch)] for _ in range(layers)]
        self.frames = [0] * layers

    def append_chunk(self, layer, chunk, pass_=0, dense=False):
        d = self.dims
        first = chunk * d.chunk_frames
        x = synth.activations(d, layer, chunk, pass_, base_seed=self.base_seed)
        wd = self.wd[layer]
        xd = to_dev(x, d)
        if dense:
            self.m.dense_append(layer, xd, wd[0], wd[1], wd[2], first, d.chunk_frames)
        else:
            self.m.append(layer, xd, wd[0], first, d.chunk_frames)
        T = d.tokens_per_frame
        for b in range(d.batch):
            for k in range(d.chunk_frames):
                self.frame_x[layer][b][first + k] = x[b, k * T:(k + 1) * T]
        self.frames[layer] = max(self.frames[layer], first + d.chunk_frames)
        return x

    def attend(self, layer, chunk, pass_=0, design=api.DESIGN_AUTO, dense=False, q_std=1.0):
        import torch
        d = self.dims
        first = chunk * d.chunk_frames
        q = synth.queries(d, layer, chunk, pass_, std=q_std, base_seed=self.base_seed)
        out = torch.full((d.batch, d.n_queries, d.n_heads * d.d_head), float("nan"), dtype=torch.float32,
                         device="cuda")
        wd = self.wd[layer]
        if dense:
            self.m.dense_attention(layer, to_dev(q, d), out, first, d.chunk_frames)
        else:
            self.m.attention(layer, to_dev(q, d), wd[1], wd[2], out, first, d.chunk_frames, design)
        st, flags = self.m.device_status()
        assert st == 0, f"device status {st} flags {flags:#x}"
        return out.float().cpu().numpy(), q

    def oracle(self, layer, chunk, q, b=0, rows=None, heads=None):
        """The fp64 definition for sample b (window rebuilt from x, window-relative positions)."""
        return oracle_chunk(self.dims, self.w[layer], self.frame_x[layer][b], chunk, q[b], rows, heads)


def oracle_chunk(d, w, frame_x, chunk, q, rows=None, heads=None):
    """fp64 output of one chunk call for one sample: ``frame_x`` maps every
    appended frame index to its x [T, d_model] (the last pass written), ``q``
    is that sample's [n_queries, n_heads, d_head]; [rows, n_heads * d_head]."""
    first = chunk * d.chunk_frames
    F = first + d.chunk_frames
    c, r, kpos, t0 = O.window_latents(frame_x, F, d.window_frames, w.w_down, d.d_latent,
                                      d.grid_h, d.grid_w, rope_at="read", sink_frames=d.sink_frames)
    qpos = O.chunk_query_positions(first, d.chunk_frames, t0, d.grid_h, d.grid_w)
    ref = O.chunk_attention(c, r, kpos, q, qpos, w.w_uk, w.w_uv, d_nope=d.d_nope, rope_pairs=d.rope_pairs,
                            rope_theta=d.rope_theta, rope_base_dims=d.rope_base_dims, query_rows=rows,
                            heads=heads)
    return ref.reshape(ref.shape[0], -1)


def sampled_rows(n_queries, count=256, seed=0):
    """``count`` seeded query rows, the last row of the call always among them."""
    rows = np.sort(np.random.default_rng(seed).choice(n_queries, min(count, n_queries), replace=False))
    rows[-1] = n_queries - 1
    return rows
