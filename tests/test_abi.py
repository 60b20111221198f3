"""The C ABI on the host: the library loads and exports every declared entry
point; configuration checks, cache accounting, RoPE frequencies, window and
frame bookkeeping.  No CUDA compute call is made here."""
import collections
import ctypes
import os
import re

import numpy as np
import pytest

import oracle.vmla_oracle as O
from latent_kv_attention_down_b200 import api, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(vmla_\w+)\s*\(", text))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    lib = api.lib()
    names = declared_functions()
    assert len(names) >= 20
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    # the binding declares a signature for each of them
    assert set(names) <= set(api._SIGS), set(names) - set(api._SIGS)


def test_abi_version_and_status_strings():
    lib = api.lib()
    assert lib.vmla_abi_version() == api.ABI_VERSION == 3
    for code in range(9):
        assert lib.vmla_status_string(code).decode().startswith("VMLA_")
    assert lib.vmla_status_string(99).decode() == "VMLA_ERR_UNKNOWN"


def default_config():
    c = api.Config()
    api.check(api.lib().vmla_config_init(ctypes.byref(c)), "init")
    return c


def test_default_config_is_the_wan_layer(golden):
    c = default_config()
    g = {k: v["value"] for k, v in golden.items()}
    assert (c.d_model, c.n_heads, c.d_latent, c.d_rope) == (g["d_model"], g["n_heads"], g["d_latent"], g["d_rope"])
    assert c.d_nope + c.d_rope == g["d_head"] and [c.d_nope, c.d_rope] == g["nope_rope_split"]
    assert list(c.rope_pairs) == g["rope_pairs_thw"]
    assert c.grid_h * c.grid_w == g["tokens_per_latent_frame"]
    assert c.window_frames == g["latent_frames_per_clip"] and c.chunk_frames == g["chunk_latent_frames"]
    assert api.lib().vmla_config_check(ctypes.byref(c)) == 0


def test_cache_bytes_match_the_pages(golden):
    """224 vs 3072 scalars per token; 3.02 B scalars / 6.0 GB for the 21-frame,
    30-layer dense cache."""
    g = {k: v["value"] for k, v in golden.items()}
    c = default_config()
    c.layers = g["layers"]
    ckv, kr, dense = api.cache_bytes(c)
    tokens = g["latent_frames_per_clip"] * g["tokens_per_latent_frame"] * g["layers"]
    assert (ckv + kr) // (2 * tokens) == g["latent_scalars_per_token"]
    assert dense // (2 * tokens) == g["dense_scalars_per_token"]
    assert round(dense / 2 / 1e9, 2) == g["dense_cache_scalars_billion"]
    assert round(dense / 1e9, 1) == g["dense_cache_gb_bf16"]
    assert round(100 * (1 - (ckv + kr) / dense), 1) == g["reduction_percent"]
    # the latent cache of one sample: 32760 tokens x 30 layers x 224 x 2 B = 0.44 GB
    assert round((ckv + kr) / 1e9, 2) == 0.44


def test_rope_frequencies_match_the_oracle():
    for base in [(0, 0, 0), (44, 42, 42)]:
        c = default_config()
        c.rope_base_dims[:] = list(base)
        got = np.array(api.rope_frequencies(c))
        ref = np.concatenate(O.rope_frequencies((6, 5, 5), 10000.0, base))
        np.testing.assert_allclose(got, ref.astype(np.float32), rtol=0, atol=0)


@pytest.mark.parametrize("field,value,status", [
    ("d_rope", 30, 1), ("rope_theta", 0.0, 1), ("batch", 0, 1), ("chunk_frames", 22, 1),
    ("grid_w", 1024, 3), ("window_frames", 1024, 3), ("d_latent", 200, 2), ("d_latent", 640, 2),
    ("d_nope", 64, 2), ("dtype", 7, 1), ("rope_mode", 3, 1),
])
def test_config_check_rejects(field, value, status):
    c = default_config()
    setattr(c, field, value)
    assert api.lib().vmla_config_check(ctypes.byref(c)) == status


@pytest.mark.parametrize("d_nope,d_rope,pairs,d_latent,status", [
    (112, 16, (4, 2, 2), 192, 0), (112, 16, (4, 2, 2), 256, 0), (64, 64, (12, 10, 10), 192, 0),
    (64, 64, (12, 10, 10), 64, 0), (64, 64, (12, 10, 10), 256, 0), (32, 96, (16, 16, 16), 128, 0),
    (32, 96, (16, 16, 16), 256, 0), (112, 16, (4, 2, 2), 384, 2), (32, 96, (16, 16, 16), 512, 2),
    (80, 48, (8, 8, 8), 192, 2),
])
def test_bf16_rotary_splits(d_nope, d_rope, pairs, d_latent, status):
    """d_head 128 split 112/16, 64/64 and 32/96 on the tensor-core path with d_latent up to 256 (the
    absorbed kernel up to 192 for 64 and 96 rotary dims); wider latents of those splits and other
    splits are refused as unsupported.  AUTO's workspace holds reconstruct-once's per-head K/V
    exactly when the full window would take it: from 192 latent dims on, or where the absorbed
    kernel does not take the split."""
    c = default_config()
    c.d_nope, c.d_rope, c.d_latent = d_nope, d_rope, d_latent
    c.rope_pairs[:] = list(pairs)
    assert api.lib().vmla_config_check(ctypes.byref(c)) == status
    if status == 0:
        recon = d_latent >= 192
        auto, absorbed = api.workspace_bytes(c, api.DESIGN_AUTO), api.workspace_bytes(c, api.DESIGN_ABSORBED)
        assert (auto > absorbed) == recon
        assert auto == api.workspace_bytes(c, api.DESIGN_RECON_ONCE if recon else api.DESIGN_ABSORBED)


def test_fp32_accepts_small_shapes():
    c = api.config_from_dims(synth.TINY)
    assert api.lib().vmla_config_check(ctypes.byref(c)) == 0


def test_workspace_bytes_grow_with_reconstruct_once():
    c = default_config()
    a = api.workspace_bytes(c, api.DESIGN_ABSORBED)
    b = api.workspace_bytes(c, api.DESIGN_RECON_ONCE)
    assert b - a >= 32760 * 3072 * 2
    assert a % 256 == 0


def test_workspace_offsets_fit_the_workspace():
    """The intermediates' regions are 256-byte aligned, disjoint and inside the workspace that
    vmla_workspace_bytes asks for: rotated keys, absorbed queries and per-head queries inside the
    base part, the per-head K/V of reconstruct-once after it."""
    c = default_config()
    off = api.workspace_offsets(c)
    T, nq = c.grid_h * c.grid_w, c.chunk_frames * c.grid_h * c.grid_w
    sizes = [c.window_frames * T * c.d_rope * 2, c.n_heads * nq * (c.d_latent + c.d_rope) * 2,
             c.n_heads * nq * (c.d_nope + c.d_rope) * 2, c.window_frames * T * 2 * c.n_heads * c.d_value * 2]
    base, full = api.workspace_bytes(c, api.DESIGN_ABSORBED), api.workspace_bytes(c, api.DESIGN_RECON_ONCE)
    assert all(o % 256 == 0 for o in off)
    spans = sorted(zip(off, sizes))
    assert all(a + n <= b for (a, n), (b, _) in zip(spans, spans[1:]))
    assert off[api.WS_QD] + sizes[api.WS_QD] <= base and off[api.WS_RECON] + sizes[api.WS_RECON] <= full
    buf = (ctypes.c_size_t * 2)()
    assert api.lib().vmla_workspace_offsets(ctypes.byref(c), buf, 2) == 1  # room for every region


def test_window_matches_a_fifo_deque():
    """vmla_window against an independent deque model of the ring, over a
    rollout of 20 chunks of 3 frames (eviction from chunk 7)."""
    h = api.LatentKVAttention(default_config())
    W = 21
    dq = collections.deque(maxlen=W)
    ring = {}
    for chunk in range(20):
        for f in range(3 * chunk, 3 * chunk + 3):
            dq.append(f)
        frames, slots, ts = h.window(3 * chunk + 3)
        assert frames == list(dq)
        assert ts == list(range(len(dq)))
        for f, s in zip(frames, slots):
            ring[s] = f
        assert all(ring[s] == f for f, s in zip(frames, slots))
        assert len(set(slots)) == len(slots)
    h.close()


def test_window_t_at_append_is_the_absolute_frame():
    """With RoPE applied at append the keys carry their absolute frame index, so vmla_window reports
    t = frame, also once the rollout has run past the ring (F > W) and the window-relative t would
    differ."""
    c = default_config()
    c.rope_mode = api.ROPE_AT_APPEND
    h = api.LatentKVAttention(c)
    for F in (3, 21, 24, 60, 300):
        frames, slots, ts = h.window(F)
        assert frames == list(range(max(0, F - 21), F))
        assert slots == [f % 21 for f in frames]
        assert ts == frames
    h.close()


def test_state_roundtrip_and_layer_range():
    c = default_config()
    c.layers = 3
    h = api.LatentKVAttention(c)
    assert h.state_get(2) == 0
    h.state_set(2, 33)
    assert h.state_get(2) == 33 and h.state_get(0) == 0
    with pytest.raises(api.VmlaError) as e:
        h.state_get(3)
    assert e.value.status == 3
    h.close()


class _FakeDev:
    """A 16-byte aligned fake device address (never dereferenced: every call
    below is rejected on the host before any launch)."""

    def __init__(self, addr):
        self.addr = addr

    def is_contiguous(self):
        return True

    def data_ptr(self):
        return self.addr


def test_frame_rule_rejections_before_any_launch():
    c = default_config()
    h = api.LatentKVAttention(c)
    lib = api.lib()
    ws = api.workspace_bytes(c)
    base = api.workspace_bytes(c, api.DESIGN_ABSORBED)  # what every design but reconstruct-once needs
    assert base < ws
    assert lib.vmla_bind(h._h, 0x10000, 0x20000, 0x30000, base - 256) == 1  # workspace too small
    assert lib.vmla_bind(h._h, 0x10008, 0x20000, 0x30000, ws) == 1        # misaligned
    assert lib.vmla_bind(h._h, 0x10000, 0x20000, 0x30000, ws) == 0
    x = w = 0x40000
    # skipping ahead or rewinding is refused
    assert lib.vmla_cache_append(h._h, 0, x, w, 3, 3, None) == 6
    assert lib.vmla_cache_append(h._h, 0, x, w, -3, 3, None) == 6
    assert lib.vmla_cache_append(h._h, 0, x, w, 0, 0, None) == 3
    assert lib.vmla_cache_append(h._h, 0, x, w, 0, 22, None) == 3
    assert lib.vmla_cache_append(h._h, 1, x, w, 0, 3, None) == 3   # layer out of range
    assert lib.vmla_cache_append(h._h, 0, 0x40008, w, 0, 3, None) == 1  # misaligned x
    # attention needs the chunk to be the newest appended frames
    assert lib.vmla_chunk_attention(h._h, 0, x, w, w, x, 0, 3, 0, None) == 6
    h.state_set(0, 9)
    assert lib.vmla_chunk_attention(h._h, 0, x, w, w, x, 3, 3, 0, None) == 6
    assert lib.vmla_chunk_attention(h._h, 0, x, w, w, x, 6, 4, 0, None) == 3   # more than chunk_frames
    assert lib.vmla_chunk_attention(h._h, 0, x, w, w, x, 6, 3, 9, None) == 1   # bad design
    assert lib.vmla_cache_append(h._h, 0, x, w, 3, 3, None) == 6              # neither new nor newest
    # the dense calls need their own cache bound first
    assert lib.vmla_dense_cache_append(h._h, 0, x, w, w, w, 0, 3, None) == 6
    assert h.state_get(0) == 9
    # the host-buffer step refuses what its append or its attention would refuse, before any copy
    step = lib.vmla_chunk_step_host
    hb = 0x50000  # host buffers: never touched when the call is refused
    assert step(h._h, 0, hb, hb, hb, w, w, w, x, x, x, 3, 3, 0, None) == 6    # skips frames
    assert step(h._h, 0, hb, hb, hb, w, w, w, x, x, x, 9, 3, 9, None) == 1    # bad design
    assert step(h._h, 0, hb, hb, hb, w, w, w, 0x40008, x, x, 9, 3, 0, None) == 1  # misaligned x_dev
    assert step(h._h, 0, hb, hb, hb, w, w, w, x, x, 0x40008, 9, 3, 0, None) == 1  # misaligned out_dev
    assert step(h._h, 1, hb, hb, hb, w, w, w, x, x, x, 9, 3, 0, None) == 3    # layer out of range
    assert h.state_get(0) == 9
    h.close()


def test_rope_at_append_range():
    c = default_config()
    c.rope_mode = api.ROPE_AT_APPEND
    h = api.LatentKVAttention(c)
    lib = api.lib()
    assert lib.vmla_bind(h._h, 0x10000, 0x20000, 0x30000, api.workspace_bytes(c)) == 0
    h.state_set(0, 1022)
    # frames 1022..1024 would put an absolute t at 1024, outside the RoPE range
    assert lib.vmla_cache_append(h._h, 0, 0x40000, 0x40000, 1022, 3, None) == 3
    h.close()


def test_append_tiling_arguments():
    c = default_config()
    h = api.LatentKVAttention(c)
    lib = api.lib()
    # (column parts, row tiles per item, grid cap); two row tiles exist only with one column part
    for t in ((3, 0, 0), (-1, 0, 0), (1, 0, -1), (0, 3, 0), (0, -1, 0), (2, 2, 0)):
        assert lib.vmla_set_append_tiling(h._h, *t) == 1, t
    for t in ((0, 0, 0), (1, 0, 0), (2, 0, 0), (1, 0, 3), (2, 0, 148), (0, 0, 7), (1, 2, 0), (0, 2, 5), (2, 1, 0)):
        assert lib.vmla_set_append_tiling(h._h, *t) == 0, t
    # one MMA covers at most 256 columns: d_latent 256 (+32) needs two column parts
    c256 = default_config()
    c256.d_latent = 256
    h2 = api.LatentKVAttention(c256)
    assert lib.vmla_bind(h2._h, 0x10000, 0x20000, 0x30000, api.workspace_bytes(c256)) == 0
    assert lib.vmla_set_append_tiling(h2._h, 1, 0, 0) == 0
    assert lib.vmla_cache_append(h2._h, 0, 0x40000, 0x40000, 0, 3, None) == 2
    for x in (h, h2):
        x.close()


def test_selftest_exp2_arguments():
    lib = api.lib()
    assert lib.vmla_selftest_exp2(0x10000, 0x20000, 3, None) == 1   # odd count
    assert lib.vmla_selftest_exp2(0x10004, 0x20000, 4, None) == 1   # misaligned
    assert lib.vmla_selftest_exp2(0, 0x20000, 4, None) == 1         # null


@pytest.mark.parametrize("d_latent,status", [(64, 0), (128, 0), (192, 0), (256, 0), (384, 0), (512, 0), (320, 2), (448, 2),
                                            (32, 2), (576, 2)])
def test_latent_widths_with_kernels(d_latent, status):
    c = default_config()
    c.d_latent = d_latent
    assert api.lib().vmla_config_check(ctypes.byref(c)) == status


@pytest.mark.parametrize("W,S,chunk", [(7, 1, 3), (7, 1, 1), (5, 2, 3), (21, 0, 3), (4, 1, 1), (9, 3, 2)])
def test_sink_window_matches_the_oracle_rule(W, S, chunk):
    """vmla_window over a 200-frame rollout: frames, ring slots and window-relative t as the oracle's
    sink rule gives them.  The t comes from the slot through the function the window-RoPE kernel
    applies to every key, so this pins the kernels' slot -> t mapping bit for bit."""
    import oracle.vmla_oracle as O
    c = default_config()
    c.window_frames, c.sink_frames, c.chunk_frames = W, S, chunk
    assert api.lib().vmla_config_check(ctypes.byref(c)) == 0
    h = api.LatentKVAttention(c)
    for F in range(1, 200):
        frames, slots, ts = h.window(F)
        want = O.window_frames_list(F, W, S)
        t = O.window_frame_t(F, W, S)
        assert list(frames) == want
        assert list(slots) == [O.ring_slot(f, W, S) for f in want]
        assert list(ts) == [t[f] for f in want]
    h.close()


def test_sink_config_rules():
    lib = api.lib()
    c = default_config()
    c.window_frames, c.sink_frames = 7, 1
    c.rope_mode = api.ROPE_AT_APPEND          # the sink context needs window-relative positions
    assert lib.vmla_config_check(ctypes.byref(c)) == 1
    c.rope_mode = api.ROPE_AT_READ
    c.sink_frames = 5                         # no room for a 3-frame chunk beside the sink
    assert lib.vmla_config_check(ctypes.byref(c)) == 1
    c.sink_frames = -1
    assert lib.vmla_config_check(ctypes.byref(c)) == 1
    c.sink_frames = 1
    h = api.LatentKVAttention(c)
    assert lib.vmla_dense_bind(h._h, 0x10000) == 2  # dense keys are rotated at absolute positions
    assert lib.vmla_bind(h._h, 0x10000, 0x20000, 0x30000, api.workspace_bytes(c)) == 0
    assert lib.vmla_cache_append(h._h, 0, 0x40000, 0x40000, 0, 7, None) == 3  # more than the local part
    h.close()
