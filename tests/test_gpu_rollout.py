"""Long rollouts at the Wan-1.3B layer shape (30x52 grid, 4680 queries, a
21-frame window of 32760 keys) through the C ABI, checked against the fp64
oracle on 256 seeded query rows of every head at chosen calls:

* 30 layers x 20 chunks x 4 sampler passes (2400 appends and 2400 chunk
  attentions): partial windows of 3..18 frames, the first eviction at chunk 7,
  every later chunk on a full ring; each pass re-writes its chunk's slots;
* checkpoint and resume: the frame counters and ring bytes copied into a
  second handle give bit-identical outputs;
* batch 8 of the same layer (8 independent rings, 30 layers, 3.52 GB of
  latent cache, 37440 queries per call).

Inputs come from a pool of seeded Gaussian frames (shifted and sign-flipped
per call) so that thousands of calls need no fresh random draws.
"""
import numpy as np
import pytest

from latent_kv_attention_down_b200 import api, synth
from tests.harness import assert_bf16_close, oracle_chunk, sampled_rows, to_dev

pytestmark = pytest.mark.gpu

WAN = synth.WAN


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


class PoolRollout:
    """One handle over ``layers`` rings fed from a FramePool on the device."""

    def __init__(self, dims, layers, pool=None, design=api.DESIGN_AUTO):
        import torch
        self.dims, self.layers, self.design = dims, layers, design
        self.pool = pool or synth.FramePool(dims)
        self.xp = to_dev(self.pool.x, dims)
        self.qp = to_dev(self.pool.q, dims)
        self.m = api.LatentKVAttention(api.config_from_dims(dims, layers)).allocate()
        self.w = {}
        self.wd = {}
        self.out = torch.empty(dims.batch, dims.n_queries, dims.n_heads * dims.d_head, dtype=torch.float32,
                               device="cuda")
        self.last_pass = {}  # (layer, chunk) -> last pass appended

    def weights(self, layer):
        if layer not in self.w:
            self.w[layer] = synth.weights(self.dims, layer)
            w = self.w[layer]
            self.wd[layer] = (to_dev(w.w_down, self.dims), to_dev(w.w_uk, self.dims), to_dev(w.w_uv, self.dims))
        return self.wd[layer]

    def step(self, layer, chunk, pass_, m=None):
        """Append the chunk's x for this pass, then attend; ``m`` overrides the handle."""
        d = self.dims
        m = m or self.m
        wd = self.weights(layer)
        first = chunk * d.chunk_frames
        m.append(layer, self.pool.activations(layer, chunk, pass_, pool=self.xp), wd[0], first, d.chunk_frames)
        m.attention(layer, self.pool.queries(layer, chunk, pass_, pool=self.qp), wd[1], wd[2], self.out, first,
                    d.chunk_frames, self.design)
        self.last_pass[(layer, chunk)] = pass_

    def check(self, layer, chunk, pass_, samples=(0,), what=""):
        """Compare the output of the call just made with the oracle on 256 rows."""
        d = self.dims
        st, flags = self.m.device_status()
        assert st == 0, f"device status {st} flags {flags:#x}"
        out = self.out.cpu().numpy()
        rows = sampled_rows(d.n_queries, 256, seed=layer * 1000 + chunk * 10 + pass_)
        T = d.tokens_per_frame
        q = self.pool.queries(layer, chunk, pass_)
        for b in samples:
            frame_x = {}
            for c in sorted({0} | set(range(max(0, chunk - d.window_frames // d.chunk_frames), chunk + 1))):
                x = self.pool.activations(layer, c, pass_ if c == chunk else self.last_pass[(layer, c)])
                for k in range(d.chunk_frames):
                    frame_x[c * d.chunk_frames + k] = x[b, k * T:(k + 1) * T]
            ref = oracle_chunk(d, self.w[layer], frame_x, chunk, q[b], rows=rows)
            assert_bf16_close(out[b][rows], ref, f"{what} layer {layer} chunk {chunk} pass {pass_} sample {b}")


@pytest.mark.parametrize("design", [api.DESIGN_AUTO, api.DESIGN_ABSORBED])
def test_wan_rollout_30_layers_20_chunks_4_passes(design):
    """AUTO runs reconstruct-once on every window of this rollout (4680 keys and more); the
    absorbed design is rolled out the same way."""
    import torch
    layers, chunks, passes = 30, 20, 4
    ro = PoolRollout(WAN, layers, design=design)
    checks = {(0, 0, 0), (17, 5, 2), (29, 6, 3), (3, 7, 0), (11, 13, 1), (29, 19, 3)}
    resume_at, resume_layers = 10, (0, 21)  # snapshot before chunk 10, replay it on a second handle
    kept = {}
    for chunk in range(chunks):
        if chunk == resume_at:
            snap = {l: ro.m.state_get(l) for l in range(layers)}
            ckv, kr = ro.m.ckv.clone(), ro.m.kr.clone()
        for p in range(passes):
            for layer in range(layers):
                ro.step(layer, chunk, p)
                if chunk == resume_at and layer in resume_layers:
                    kept[(layer, p)] = ro.out.clone()
                if (layer, chunk, p) in checks:
                    ro.check(layer, chunk, p, what="rollout")
        assert all(ro.m.state_get(l) == (chunk + 1) * WAN.chunk_frames for l in range(layers))
    # resume: the frame counters and the ring bytes alone carry the state -> bit-identical outputs
    m2 = api.LatentKVAttention(api.config_from_dims(WAN, layers))
    m2.bind(ckv, kr, torch.empty_like(ro.m.workspace))
    for l, f in snap.items():
        m2.state_set(l, f)
    for layer in resume_layers:
        for p in range(passes):
            ro.step(layer, resume_at, p, m=m2)
            assert torch.equal(ro.out, kept[(layer, p)]), f"resumed layer {layer} pass {p} differs"
    assert m2.device_status()[0] == 0


def test_wan_batch8_sampled_rows():
    d = WAN.replace(batch=8)
    layers = 30
    ro = PoolRollout(d, layers)
    for layer in (0, 13, 29):
        for chunk in range(7):
            ro.step(layer, chunk, 0)
        if layer == 13:
            continue
        ro.check(layer, 6, 0, samples=(0, 5) if layer == 0 else (3, 7), what="batch 8")


@pytest.mark.parametrize("d_latent", [64, 128, 192, 256, 384, 512])
def test_wan_latent_width_sweep(d_latent):
    """The Wan-1.3B layer with latent widths 64..256 (same seeded x and q), every
    built design and the dense per-head cache, on 256 rows of every head."""
    from tests.harness import Rollout
    d = WAN.replace(d_latent=d_latent)
    ro = Rollout(d, design=api.DESIGN_RECON_ONCE, dense=True)  # workspace sized for every design
    for c in range(7):
        ro.append_chunk(0, c)
        ro.append_chunk(0, c, dense=True)
    rows = sampled_rows(d.n_queries, 256, seed=d_latent)
    got = {}
    designs = [("recon_once", api.DESIGN_RECON_ONCE)]
    if d_latent <= 256:
        designs.append(("absorbed", api.DESIGN_ABSORBED))
    if d_latent <= 192:
        designs.append(("reconstruct_in_tile", api.DESIGN_RECONSTRUCT))
    for name, design in designs:
        out, q = ro.attend(0, 6, design=design)
        got[name] = out[0][rows]
    out, q = ro.attend(0, 6, dense=True)
    got["dense"] = out[0][rows]
    ref = ro.oracle(0, 6, q, rows=rows)
    for name, o in got.items():
        assert_bf16_close(o, ref, f"{name} d_c={d_latent}")


def test_wan_sink_window_sampled_rows():
    """The Wan layer in the pages' long-horizon context (one sink frame + six
    recent frames: 10920 keys) after 12 chunks, 256 seeded rows of every head."""
    d = synth.WAN_SINK
    ro = PoolRollout(d, 1)
    for chunk in range(12):
        ro.step(0, chunk, 0)
    ro.check(0, 11, 0, what="sink window")


def test_wan_folded_output_mixer_sampled_rows():
    """The folded output mixer at the Wan layer shape (K = 12 x 192, d_out = 1536)."""
    import torch
    import oracle.vmla_oracle as O
    d = WAN
    ro = PoolRollout(d, 1)
    for chunk in range(7):
        ro.step(0, chunk, 0)
    w = ro.w[0]
    w_fold = torch.empty(d.d_model, d.n_heads * d.d_latent, dtype=torch.bfloat16, device="cuda")
    ro.m.fold_output_weights(to_dev(w.w_o, d), ro.wd[0][2], w_fold)
    out = torch.empty(1, d.n_queries, d.d_model, dtype=torch.float32, device="cuda")
    ro.m.attention_folded(0, ro.pool.queries(0, 6, 0, pool=ro.qp), ro.wd[0][1], w_fold, out, 18, 3)
    assert ro.m.device_status()[0] == 0
    rows = sampled_rows(d.n_queries, 256, seed=5)
    frame_x = {}
    T = d.tokens_per_frame
    for c in range(7):
        x = ro.pool.activations(0, c, 0)
        for k in range(d.chunk_frames):
            frame_x[c * d.chunk_frames + k] = x[0, k * T:(k + 1) * T]
    heads = oracle_chunk(d, w, frame_x, 6, ro.pool.queries(0, 6, 0)[0], rows=rows)
    ref = O.output_projection(heads.reshape(len(rows), d.n_heads, d.d_head), w.w_o)
    assert_bf16_close(out[0].cpu().numpy()[rows], ref, "folded output mixer, Wan layer")
