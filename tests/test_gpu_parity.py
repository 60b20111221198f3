"""CUDA path vs the fp64 oracle, through the C ABI, on seeded inputs.

Workloads: the tiny fp32 layer (SIMT kernels, relative L2 <= 1e-5); the
Wan-1.3B layer on a 10x20 grid (tcgen05 kernels; several query and key tiles
with ragged tails; full comparison at the bf16 gate: relative L2 <= 1e-2 and
max |err| <= 3e-2 RMS); the full Wan-1.3B layer (30x52 grid, 4680 queries,
32760 keys) on seeded query rows.
"""
import numpy as np
import pytest

from latent_kv_attention_down_b200 import api, synth
from tests.harness import Rollout, assert_bf16_close, assert_fp32_close, sampled_rows, to_dev

pytestmark = pytest.mark.gpu

TINY, SMALL, WAN = synth.TINY, synth.WAN_SMALL, synth.WAN


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


# ------------------------------------------------------------------ tiny fp32 (SIMT)

@pytest.mark.parametrize("rope_mode", [api.ROPE_AT_READ, api.ROPE_AT_APPEND])
def test_tiny_fp32_rolling_window(rope_mode):
    """9 one-frame chunks through a 4-frame ring: partial windows, eviction,
    wrap-around; every chunk checked in full."""
    ro = Rollout(TINY, rope_mode=rope_mode)
    for chunk in range(9):
        ro.append_chunk(0, chunk)
        out, q = ro.attend(0, chunk)
        assert_fp32_close(out[0], ro.oracle(0, chunk, q), f"chunk {chunk}")


def test_tiny_fp32_denoising_passes_rewrite_the_chunk():
    ro = Rollout(TINY)
    for chunk in range(6):
        for p in range(4):  # 4 sampler passes: each re-appends the chunk, then attends
            ro.append_chunk(0, chunk, pass_=p)
            out, q = ro.attend(0, chunk, pass_=p)
            assert_fp32_close(out[0], ro.oracle(0, chunk, q), f"chunk {chunk} pass {p}")


def test_tiny_fp32_dense():
    ro = Rollout(TINY, dense=True)
    for chunk in range(7):
        ro.append_chunk(0, chunk, dense=True)
        out, q = ro.attend(0, chunk, dense=True)
        assert_fp32_close(out[0], ro.oracle(0, chunk, q), f"dense chunk {chunk}")


@pytest.mark.parametrize("d_nope,d_rope,pairs", [(112, 16, (4, 2, 2)), (64, 64, (12, 10, 10)),
                                                 (32, 96, (18, 15, 15))])
def test_fp32_nope_rope_split_variants(d_nope, d_rope, pairs):
    """Other splits of a 128-dim head between content and positional dims (16, 64 and 96
    rotary dims) through the fp32 kernels, rolling past the window."""
    d = TINY.replace(name=f"split{d_rope}", d_model=64, n_heads=2, d_nope=d_nope, d_rope=d_rope, d_latent=16,
                     rope_pairs=pairs)
    ro = Rollout(d)
    for chunk in range(6):
        ro.append_chunk(0, chunk)
        out, q = ro.attend(0, chunk)
        assert_fp32_close(out[0], ro.oracle(0, chunk, q), f"d_rope {d_rope} chunk {chunk}")


def test_tiny_fp32_batch_and_layers():
    d = TINY.replace(batch=3)
    ro = Rollout(d, layers=2)
    for chunk in range(5):
        for layer in range(2):
            ro.append_chunk(layer, chunk)
            out, q = ro.attend(layer, chunk)
            for b in range(3):
                assert_fp32_close(out[b], ro.oracle(layer, chunk, q, b), f"layer {layer} sample {b}")


# ------------------------------------------------------------------ bf16 tcgen05, 10x20 grid

def _fill(ro, chunks, layer=0, dense=False):
    for c in range(chunks):
        ro.append_chunk(layer, c, dense=dense)


@pytest.mark.parametrize("chunks", [1, 2, 7, 10])
def test_small_bf16_absorbed(chunks):
    """1 chunk (600 keys, one query frame set), 2 (partial window), 7 (full
    21-frame window, 4200 keys), 10 (evicted, wrapped ring)."""
    ro = Rollout(SMALL)
    _fill(ro, chunks)
    out, q = ro.attend(0, chunks - 1, design=api.DESIGN_ABSORBED)
    assert_bf16_close(out[0], ro.oracle(0, chunks - 1, q), f"{chunks} chunks")


@pytest.mark.parametrize("chunks", [7, 10])
def test_small_bf16_auto(chunks):
    """AUTO on the full 21-frame window (4200 keys: reconstruct-once) and on the wrapped ring."""
    ro = Rollout(SMALL)
    _fill(ro, chunks)
    out, q = ro.attend(0, chunks - 1)
    assert_bf16_close(out[0], ro.oracle(0, chunks - 1, q), f"AUTO, {chunks} chunks")


@pytest.mark.parametrize("design,dense", [(api.DESIGN_ABSORBED, False), (api.DESIGN_RECON_ONCE, False),
                                          (api.DESIGN_AUTO, True)])
def test_small_bf16_forced_rescale(design, dense):
    """Threshold 0: the running max is raised (and O rescaled in TMEM) at every
    increase, so the correction path runs many times per row."""
    ro = Rollout(SMALL, rescale_log2=0.0, dense=dense, design=api.DESIGN_RECON_ONCE)
    _fill(ro, 8, dense=dense)
    out, q = ro.attend(0, 7, design=design, dense=dense)
    assert_bf16_close(out[0], ro.oracle(0, 7, q), "forced rescale")


@pytest.mark.parametrize("design", [api.DESIGN_ABSORBED, api.DESIGN_RECON_ONCE])
def test_small_bf16_rope_at_append(design):
    ro = Rollout(SMALL, rope_mode=api.ROPE_AT_APPEND)
    _fill(ro, 9)
    out, q = ro.attend(0, 8, design=design)
    assert_bf16_close(out[0], ro.oracle(0, 8, q), "rope at append")


@pytest.mark.parametrize("design", [api.DESIGN_ABSORBED, api.DESIGN_AUTO])
def test_small_bf16_denoising_passes(design):
    ro = Rollout(SMALL)
    _fill(ro, 7)
    for p in range(4):
        ro.append_chunk(0, 7, pass_=p)
        out, q = ro.attend(0, 7, pass_=p, design=design)
        assert_bf16_close(out[0], ro.oracle(0, 7, q), f"pass {p}")


def test_small_bf16_dense():
    ro = Rollout(SMALL, dense=True)
    _fill(ro, 8, dense=True)
    out, q = ro.attend(0, 7, dense=True)
    assert_bf16_close(out[0], ro.oracle(0, 7, q), "dense")


def test_small_bf16_reconstruct_once():
    ro = Rollout(SMALL, design=api.DESIGN_RECON_ONCE)
    _fill(ro, 8)
    out, q = ro.attend(0, 7, design=api.DESIGN_RECON_ONCE)
    assert_bf16_close(out[0], ro.oracle(0, 7, q), "reconstruct once")


@pytest.mark.parametrize("d_latent", [64, 128, 256, 384, 512])
def test_small_bf16_latent_width(d_latent):
    """The design AUTO picks (absorbed up to 192, reconstruct-once above) at the gate."""
    ro = Rollout(SMALL.replace(name=f"small_dc{d_latent}", d_latent=d_latent))
    _fill(ro, 8)
    out, q = ro.attend(0, 7)
    assert_bf16_close(out[0], ro.oracle(0, 7, q), f"d_latent {d_latent}")


@pytest.mark.parametrize("chunks", [1, 3, pytest.param(8, marks=pytest.mark.xfail(
    strict=True, reason="fails the max-error gate (3.4e-2 RMS): the absorbed query's bf16 rounding at 256 "
                        "latent dims; AUTO takes reconstruct-once there"))])
def test_small_bf16_absorbed_at_latent_256(chunks):
    """The absorbed design at d_latent = 256 (its bf16 query, one rounding per row reused against
    every key, adds a coherent score error to the cache's) on short, mid and full windows."""
    ro = Rollout(SMALL.replace(name="small_dc256", d_latent=256), design=api.DESIGN_ABSORBED)
    _fill(ro, chunks)
    out, q = ro.attend(0, chunks - 1, design=api.DESIGN_ABSORBED)
    assert_bf16_close(out[0], ro.oracle(0, chunks - 1, q), f"absorbed d_c 256, {chunks} chunks")


def test_small_bf16_batch_and_layers():
    d = SMALL.replace(name="small_b2", batch=2)
    ro = Rollout(d, layers=2)
    for c in range(8):
        for layer in range(2):
            ro.append_chunk(layer, c)
    for layer in range(2):
        out, q = ro.attend(layer, 7)
        for b in range(2):
            assert_bf16_close(out[b], ro.oracle(layer, 7, q, b), f"layer {layer} sample {b}")


# Per-head designs that round each key's K_h and V_h to bf16 (reconstruct-in-tile and the dense
# comparison, whose cache is bf16 by definition) fail the max-error gate on the shortest window:
# over 600 keys the per-key roundings do not average out (measured 4.55e-2 RMS on these inputs;
# relative L2 2.8e-3 passes).  These cases are kept as strict expected failures at the gate, next
# to the stage-wise checks that hold the same kernels to their own rounding bounds.
SHORT_WINDOW_FAILS = pytest.mark.xfail(strict=True, reason="fails the max-error gate on a 600-key window: "
                                                          "bf16 rounding of every key's per-head K and V")


@pytest.mark.parametrize("chunks", [pytest.param(1, marks=SHORT_WINDOW_FAILS), 2, 7, 10])
def test_small_bf16_reconstruct_in_tile(chunks):
    """Design (b): per-head K/V rebuilt from the latent tile on the tensor core
    inside the attention kernel; partial window, full window, wrapped ring."""
    ro = Rollout(SMALL)
    _fill(ro, chunks)
    out, q = ro.attend(0, chunks - 1, design=api.DESIGN_RECONSTRUCT)
    assert_bf16_close(out[0], ro.oracle(0, chunks - 1, q), f"reconstruct, {chunks} chunks")


@pytest.mark.parametrize("d_latent", [64, 128])
def test_small_bf16_reconstruct_in_tile_latent_width(d_latent):
    d = SMALL.replace(d_latent=d_latent)
    ro = Rollout(d)
    _fill(ro, 8)
    out, q = ro.attend(0, 7, design=api.DESIGN_RECONSTRUCT)
    assert_bf16_close(out[0], ro.oracle(0, 7, q), f"reconstruct d_c={d_latent}")


def test_small_bf16_reconstruct_in_tile_rope_at_append_and_rescale():
    ro = Rollout(SMALL, rope_mode=api.ROPE_AT_APPEND, rescale_log2=0.0)
    _fill(ro, 8)
    out, q = ro.attend(0, 7, design=api.DESIGN_RECONSTRUCT)
    assert_bf16_close(out[0], ro.oracle(0, 7, q), "reconstruct, rope at append, rescale every tile")


@pytest.mark.parametrize("design,dense", [(api.DESIGN_RECON_ONCE, False),
                                          pytest.param(api.DESIGN_RECONSTRUCT, False, marks=SHORT_WINDOW_FAILS),
                                          pytest.param(api.DESIGN_AUTO, True, marks=SHORT_WINDOW_FAILS)])
def test_small_bf16_per_head_designs_short_window(design, dense):
    """The per-head designs on a 600-key window (the first chunk): reconstruct-once, whose per-head
    K, V, queries and probabilities are fp16, meets the gate; the bf16 per-head tiles of
    reconstruct-in-tile and of the dense cache do not."""
    ro = Rollout(SMALL, design=api.DESIGN_RECON_ONCE, dense=dense)
    ro.append_chunk(0, 0, dense=dense)
    out, q = ro.attend(0, 0, design=design, dense=dense)
    assert_bf16_close(out[0], ro.oracle(0, 0, q), f"design {design} dense {dense}")


# content/rotary splits of a 128-dim head [paperlayer App. F]: 112/16, 96/32, 64/64, 32/96, with the
# rotary pairs split over (t, h, w) as (4,2,2), (6,5,5), (12,10,10), (16,16,16)
SPLITS = {16: (112, (4, 2, 2)), 64: (64, (12, 10, 10)), 96: (32, (16, 16, 16))}


def split_dims(base, d_rope, d_latent=192):
    d_nope, pairs = SPLITS[d_rope]
    return base.replace(name=f"{base.name}_r{d_rope}_c{d_latent}", d_nope=d_nope, d_rope=d_rope, rope_pairs=pairs,
                        d_latent=d_latent)


SPLIT_WINDOWS = [(192, 2), (192, 7), (192, 10), (64, 7), (128, 7), (256, 7)]


def _split_rollout(d_rope, d_latent, chunks, dense):
    d = split_dims(SMALL, d_rope, d_latent)
    ro = Rollout(d, design=api.DESIGN_RECON_ONCE, dense=dense)
    for c in range(chunks):
        ro.append_chunk(0, c, dense=dense)
    return d, ro


@pytest.mark.parametrize("d_rope", [16, 64, 96])
@pytest.mark.parametrize("d_latent,chunks", SPLIT_WINDOWS)
def test_small_bf16_rotary_split_reconstruct_once_and_auto(d_rope, d_latent, chunks):
    """Every content/rotary split through reconstruct-once (fp16 per-head operands) and through
    the design AUTO takes: partial, full and wrapped windows, in full, at the gate."""
    d, ro = _split_rollout(d_rope, d_latent, chunks, dense=False)
    ref = None
    for name, design in (("recon_once", api.DESIGN_RECON_ONCE), ("auto", api.DESIGN_AUTO)):
        out, q = ro.attend(0, chunks - 1, design=design)
        if ref is None:
            ref = ro.oracle(0, chunks - 1, q)
        assert_bf16_close(out[0], ref, f"{d.d_nope}/{d_rope}, d_c {d_latent}, {chunks} chunks, {name}")


# Where the max-error gate fails for the designs that round per row or per key to bf16 (the absorbed
# query q~; every key's per-head K and V in the dense cache), measured on these seeded inputs; the
# stage-wise tests hold the same kernels to their own rounding bounds.
def _gate_fails(reason):
    return pytest.mark.xfail(strict=True, reason="fails the max-error gate: " + reason)


DENSE_FAILS = {(96, 192, 10)}


@pytest.mark.parametrize("d_rope,d_latent,chunks", [
    pytest.param(r, dl, ch, marks=_gate_fails("bf16 per-head cache entries") if (r, dl, ch) in DENSE_FAILS else ())
    for r in (16, 64, 96) for dl, ch in SPLIT_WINDOWS])
def test_small_bf16_rotary_split_dense_cache(d_rope, d_latent, chunks):
    """The dense per-head cache (bf16 K/V per head and key) with every content/rotary split."""
    d, ro = _split_rollout(d_rope, d_latent, chunks, dense=True)
    out, q = ro.attend(0, chunks - 1, dense=True)
    assert_bf16_close(out[0], ro.oracle(0, chunks - 1, q), f"{d.d_nope}/{d_rope}, d_c {d_latent}, {chunks}, dense")


ABSORBED_FAILS = {(96, 192, 2), (96, 192, 10)}  # 3.2e-2 and 4.0e-2 RMS: 96 rotary dims leave 32 content dims


@pytest.mark.parametrize("d_rope,d_latent,chunks", [
    pytest.param(r, dl, ch, marks=_gate_fails("the absorbed query's bf16 rounding") if (r, dl, ch) in ABSORBED_FAILS
                 else ())
    for r in (16, 64, 96) for dl, ch in SPLIT_WINDOWS if r == 16 or dl <= 192])
def test_small_bf16_rotary_split_absorbed(d_rope, d_latent, chunks):
    """The absorbed kernel with every content/rotary split it takes (rotary blocks swizzled at their
    width; 96 dims as three 32-column blocks; 64 and 96 up to d_latent 192)."""
    d, ro = _split_rollout(d_rope, d_latent, chunks, dense=False)
    out, q = ro.attend(0, chunks - 1, design=api.DESIGN_ABSORBED)
    assert_bf16_close(out[0], ro.oracle(0, chunks - 1, q), f"{d.d_nope}/{d_rope}, d_c {d_latent}, {chunks}, absorbed")


@pytest.mark.parametrize("d_rope", [16, 64, 96])
def test_rotary_split_reconstruct_in_tile_refused(d_rope):
    """Reconstruct-in-tile keeps the 96/32 split; the others return VMLA_ERR_UNSUPPORTED_SHAPE, and
    the absorbed design refuses 64 and 96 rotary dims past d_latent 192."""
    d = split_dims(SMALL, d_rope)
    ro = Rollout(d)
    _fill(ro, 1)
    with pytest.raises(api.VmlaError, match="UNSUPPORTED"):
        ro.attend(0, 0, design=api.DESIGN_RECONSTRUCT)
    if d_rope != 16:
        ro = Rollout(split_dims(SMALL, d_rope, 256))
        _fill(ro, 1)
        with pytest.raises(api.VmlaError, match="UNSUPPORTED"):
            ro.attend(0, 0, design=api.DESIGN_ABSORBED)


@pytest.mark.parametrize("d_rope", [16, 64, 96])
def test_wan_layer_rotary_split_every_design(d_rope):
    """The Wan-1.3B layer with each split (4680 queries over 32760 keys), 256 seeded rows of every
    head, for the absorbed design, reconstruct-once (what AUTO takes) and the dense cache."""
    d = split_dims(WAN, d_rope)
    ro = Rollout(d, design=api.DESIGN_RECON_ONCE, dense=True)
    for c in range(7):
        ro.append_chunk(0, c)
        ro.append_chunk(0, c, dense=True)
    rows = sampled_rows(d.n_queries, 256, seed=d_rope)
    ref = None
    for name, design, dense in (("absorbed", api.DESIGN_ABSORBED, False), ("auto", api.DESIGN_AUTO, False),
                                ("dense", api.DESIGN_AUTO, True)):
        out, q = ro.attend(0, 6, design=design, dense=dense)
        if ref is None:
            ref = ro.oracle(0, 6, q, rows=rows)
        assert_bf16_close(out[0][rows], ref, f"Wan layer {d.d_nope}/{d_rope}, {name}")


def test_absorbed_rejects_latent_384():
    d = SMALL.replace(d_latent=384)
    ro = Rollout(d)
    _fill(ro, 1)
    with pytest.raises(api.VmlaError, match="UNSUPPORTED"):
        ro.attend(0, 0, design=api.DESIGN_ABSORBED)


def test_reconstruct_in_tile_rejects_latent_256():
    d = SMALL.replace(d_latent=256)
    ro = Rollout(d)
    _fill(ro, 1)
    with pytest.raises(api.VmlaError, match="UNSUPPORTED"):
        ro.attend(0, 0, design=api.DESIGN_RECONSTRUCT)


def test_small_append_writes_only_its_slots():
    """Ring rows of the appended frames hold bf16(W_down x) (bf16 rounding of
    the fp64 product); every other byte of the cache is untouched."""
    import torch
    import oracle.vmla_oracle as O
    ro = Rollout(SMALL)
    ro.m.ckv.fill_(0x7F)
    ro.m.kr.fill_(0x7F)
    ro.append_chunk(0, 0)
    ro.append_chunk(0, 1)
    torch.cuda.synchronize()
    d = SMALL
    T = d.tokens_per_frame
    ckv = ro.m.ckv.view(torch.bfloat16).view(d.window_frames * T, d.d_latent).float().cpu().numpy()
    kr = ro.m.kr.view(torch.bfloat16).view(d.window_frames * T, d.d_rope).float().cpu().numpy()
    x = np.concatenate([ro.frame_x[0][0][f] for f in range(6)])
    c, r = O.down_project(x, ro.w[0].w_down, d.d_latent)
    for got, ref in ((ckv[:6 * T], c), (kr[:6 * T], r)):
        err = np.abs(got - ref)
        assert np.all(err <= 2.0 ** -8 * np.abs(ref) + 1e-6 * np.abs(ref).max()), err.max()
    raw_ckv = ro.m.ckv.view(d.window_frames * T, -1)[6 * T:].cpu().numpy()
    raw_kr = ro.m.kr.view(d.window_frames * T, -1)[6 * T:].cpu().numpy()
    assert np.all(raw_ckv == 0x7F) and np.all(raw_kr == 0x7F)


# (column parts, 128-row tiles per item, grid cap)
TILINGS = [(0, 0, 0), (1, 1, 0), (2, 0, 0), (1, 1, 1), (2, 0, 3), (1, 2, 0), (1, 2, 3), (1, 2, 1)]


@pytest.mark.parametrize("tiling", TILINGS, ids=lambda t: "np%d_mt%d_ctas%d" % t)
@pytest.mark.parametrize("rope_mode", [api.ROPE_AT_READ, api.ROPE_AT_APPEND])
def test_append_tilings(tiling, rope_mode):
    """Every work split of the persistent append kernel (one or two column
    parts; one or two row tiles per item, a pair crossing from one sample's
    ragged last tile into the next sample and the last item holding a single
    tile; a grid of one CTA per SM, or capped so each CTA runs many items
    through its TMEM accumulators) writes bf16(W_down x) -- k_R rotated with the
    absolute frame when RoPE is applied at append -- into exactly its ring rows,
    for three samples and a ragged last tile (600 rows per sample: 5 tiles)."""
    import torch
    import oracle.vmla_oracle as O
    d = SMALL.replace(name="small_b3", batch=3)
    ro = Rollout(d, rope_mode=rope_mode)
    ro.m.set_append_tiling(*tiling)
    ro.m.ckv.fill_(0x7F)
    ro.m.kr.fill_(0x7F)
    for c in range(3):  # frames 0..8; the ring holds 21
        ro.append_chunk(0, c)
    torch.cuda.synchronize()
    assert ro.m.device_status()[0] == 0
    T, R = d.tokens_per_frame, d.window_frames * d.tokens_per_frame
    n = 9 * T
    ckv = ro.m.ckv.view(torch.bfloat16).view(d.batch, R, d.d_latent).float().cpu().numpy()
    kr = ro.m.kr.view(torch.bfloat16).view(d.batch, R, d.d_rope).float().cpu().numpy()
    freqs = O.rope_frequencies(d.rope_pairs, d.rope_theta, d.rope_base_dims)
    pos = O.key_positions(range(9), 0, d.grid_h, d.grid_w)
    for b in range(d.batch):
        x = np.concatenate([ro.frame_x[0][b][f] for f in range(9)])
        c, r = O.down_project(x, ro.w[0].w_down, d.d_latent)
        if rope_mode == api.ROPE_AT_APPEND:
            r = O.rope_rotate(r, O.rope_angles(pos[:, 0], pos[:, 1], pos[:, 2], freqs))
        for got, ref, what in ((ckv[b, :n], c, "c_KV"), (kr[b, :n], r, "k_R")):
            err = np.abs(got - ref)
            bound = 2.0 ** -8 * np.abs(ref) + 1e-5 * np.abs(ref).max()
            assert np.all(err <= bound), f"{what} sample {b}: worst excess {np.max(err - bound):.3e}"
    raw_ckv = ro.m.ckv.view(d.batch, R, -1)[:, n:].cpu().numpy()
    raw_kr = ro.m.kr.view(d.batch, R, -1)[:, n:].cpu().numpy()
    assert np.all(raw_ckv == 0x7F) and np.all(raw_kr == 0x7F)


# The tiny layer (d_model 32, 2 heads of 10 + 6, d_c 8, rotary pairs (1, 1, 1), a 4x6
# grid, a 4-frame window of 1-frame chunks: 96 keys, 24 queries) zero-padded into the
# widths the tensor-core kernels take: d_model 64, d_c 64, heads of 96 + 32 with the
# rotary pairs (14, 1, 1).  The first pair of every axis turns at theta^0 = 1 whatever
# the band size, so the tiny layer's three pairs become pairs 0, 14 and 15 of the
# padded head and every other pair carries zeros.  Every tile is mostly padding: the
# TMA zero fill past the last key and query and the ragged-tile masks decide the result.
TINY_BF16 = TINY.replace(dtype="bf16")
TINY_PADDED = TINY.replace(name="tiny_padded", d_model=64, d_nope=96, d_rope=32, d_latent=64,
                           rope_pairs=(14, 1, 1), dtype="bf16")
_PAD_PAIR = (0, 14, 15)  # padded pair of each of the tiny layer's (t, h, w) pairs


def _pad_rotary(dst, src):
    """Tiny rotary pairs [..., 6] into the padded [..., 32] layout."""
    for k, p in enumerate(_PAD_PAIR):
        dst[..., 2 * p:2 * p + 2] = src[..., 2 * k:2 * k + 2]


@pytest.mark.parametrize("design", [api.DESIGN_AUTO, api.DESIGN_ABSORBED, api.DESIGN_RECON_ONCE,
                                    api.DESIGN_RECONSTRUCT])
def test_tiny_layer_zero_padded_through_tensor_cores(design):
    """The tiny layer, zero-padded, through the bf16 tensor-core kernels over a
    rollout that wraps the ring (chunk 6 of 1-frame chunks, 4-frame window),
    against the fp64 definition of the unpadded layer; the padded value columns
    come out exactly zero.  The softmax scale of the padded head is
    1/sqrt(128) against the tiny head's 1/sqrt(16): the padded queries carry
    the factor sqrt(8), and the oracle takes them divided back."""
    import torch
    from tests.harness import oracle_chunk
    t, d = TINY_BF16, TINY_PADDED
    w = synth.weights(t, 0)
    wd = np.zeros((d.d_latent + d.d_rope, d.d_model), np.float32)
    wd[:t.d_latent, :t.d_model] = w.w_down[:t.d_latent]
    _pad_rotary(wd[d.d_latent:, :t.d_model].T, w.w_down[t.d_latent:].T)
    wuk = np.zeros((d.n_heads, d.d_nope, d.d_latent), np.float32)
    wuk[:, :t.d_nope, :t.d_latent] = w.w_uk
    wuv = np.zeros((d.n_heads, d.d_head, d.d_latent), np.float32)
    wuv[:, :t.d_head, :t.d_latent] = w.w_uv
    cfg = api.config_from_dims(d)
    m = api.LatentKVAttention(cfg).allocate(design=design)
    W = [to_dev(a, d) for a in (wd, wuk, wuv)]
    frame_x = {}
    chunk = 6
    for c in range(chunk + 1):
        x = synth.activations(t, 0, c)
        xp = np.zeros((1, x.shape[1], d.d_model), np.float32)
        xp[..., :t.d_model] = x
        m.append(0, to_dev(xp, d), W[0], c, 1)
        frame_x[c] = x[0]
    s8 = np.float32(np.sqrt(8.0))
    q = synth.queries(t, 0, chunk)
    qp = np.zeros((1, q.shape[1], d.n_heads, d.d_head), np.float32)
    qp[..., :t.d_nope] = q[..., :t.d_nope] * s8
    _pad_rotary(qp[..., d.d_nope:], q[..., t.d_nope:] * s8)
    qp_dev = to_dev(qp, d)
    out = torch.full((1, d.n_queries, d.n_heads * d.d_head), float("nan"), dtype=torch.float32, device="cuda")
    m.attention(0, qp_dev, W[1], W[2], out, chunk, 1, design)
    st, flags = m.device_status()
    assert st == 0, f"device status {st} flags {flags:#x}"
    got = out.cpu().numpy().reshape(d.n_queries, d.n_heads, d.d_head)
    m.close()
    qb = qp_dev.float().cpu().numpy().astype(np.float64) / np.sqrt(8.0)  # the padded queries as stored, rescaled
    q_oracle = np.concatenate([qb[0, :, :, :t.d_nope],
                               np.stack([qb[0, :, :, d.d_nope + 2 * p + e] for p in _PAD_PAIR for e in (0, 1)],
                                        axis=-1)], axis=-1)
    ref = oracle_chunk(t, w, frame_x, chunk, q_oracle).reshape(t.n_queries, t.n_heads, t.d_head)
    assert np.all(got[:, :, t.d_head:] == 0), "padded value columns"
    assert_bf16_close(got[:, :, :t.d_head].reshape(t.n_queries, -1), ref.reshape(t.n_queries, -1),
                      f"tiny layer zero-padded, design {design}")


@pytest.mark.parametrize("tiling", [(1, 1, 0), (2, 0, 0), (2, 0, 1), (1, 2, 1)], ids=lambda t: "np%d_mt%d_ctas%d" % t)
def test_small_bf16_attention_after_tiled_appends(tiling):
    """The full path with a forced append tiling, against the oracle."""
    ro = Rollout(SMALL)
    ro.m.set_append_tiling(*tiling)
    _fill(ro, 8)
    out, q = ro.attend(0, 7)
    assert_bf16_close(out[0], ro.oracle(0, 7, q), f"tiling {tiling}")


@pytest.mark.parametrize("design", [api.DESIGN_ABSORBED, api.DESIGN_RECON_ONCE, api.DESIGN_RECONSTRUCT])
def test_small_output_rows_and_guards(design):
    """Attention writes exactly its output tensor: guard rows around it stay
    bit-identical."""
    import torch
    ro = Rollout(SMALL, design=api.DESIGN_RECON_ONCE)
    _fill(ro, 8)
    d = SMALL
    q = synth.queries(d, 0, 7)
    width = d.n_heads * d.d_head
    buf = torch.full((d.n_queries + 64, width), 12345.0, dtype=torch.float32, device="cuda")
    out = buf[32:32 + d.n_queries]
    ro.m.attention(0, to_dev(q, d), ro.wd[0][1], ro.wd[0][2], out, 21, 3, design)
    assert ro.m.device_status()[0] == 0
    b = buf.float().cpu().numpy()
    assert np.all(b[:32] == 12345.0) and np.all(b[32 + d.n_queries:] == 12345.0)
    assert_bf16_close(b[32:32 + d.n_queries], ro.oracle(0, 7, q), "guarded")


def test_step_host_matches_device_path():
    import torch
    ro = Rollout(SMALL)
    _fill(ro, 7)
    d = SMALL
    x = synth.activations(d, 0, 7)
    q = synth.queries(d, 0, 7)
    xh = torch.from_numpy(x).to(torch.bfloat16).pin_memory()
    qh = torch.from_numpy(q).to(torch.bfloat16).pin_memory()
    oh = torch.empty((1, d.n_queries, d.n_heads * d.d_head), dtype=torch.float32).pin_memory()
    xd, qd = torch.empty_like(xh, device="cuda"), torch.empty_like(qh, device="cuda")
    od = torch.empty_like(oh, device="cuda")
    wd = ro.wd[0]
    ro.m.step_host(0, xh, qh, oh, wd[0], wd[1], wd[2], xd, qd, od, 21, 3)
    torch.cuda.synchronize()
    ro.frame_x[0][0].update({21 + k: x[0, k * d.tokens_per_frame:(k + 1) * d.tokens_per_frame] for k in range(3)})
    assert_bf16_close(oh.float().numpy()[0], ro.oracle(0, 7, q), "host step")


@pytest.mark.parametrize("design", [api.DESIGN_AUTO, api.DESIGN_ABSORBED])
def test_step_host_head_groups_match_device_path(design):
    """Batch 4 on the small grid: the host-buffer step runs the attention as one launch per group
    of heads that fills the GPU once (7 + 5 heads) and copies each group's output columns back
    while the next group computes.  Two consecutive calls on the same staging buffers, issued
    without a wait between them, must equal the device path bit for bit."""
    import torch
    d = SMALL.replace(batch=4)
    dev, host = Rollout(d), Rollout(d)
    _fill(dev, 6)
    _fill(host, 6)
    xd = torch.empty((d.batch, d.n_queries, d.d_model), dtype=torch.bfloat16, device="cuda")
    qd = torch.empty((d.batch, d.n_queries, d.n_heads, d.d_head), dtype=torch.bfloat16, device="cuda")
    od = torch.empty((d.batch, d.n_queries, d.n_heads * d.d_head), dtype=torch.float32, device="cuda")
    keep, outs = [], []
    for chunk in (6, 7):
        x = torch.from_numpy(synth.activations(d, 0, chunk)).to(torch.bfloat16).pin_memory()
        q = torch.from_numpy(synth.queries(d, 0, chunk)).to(torch.bfloat16).pin_memory()
        oh = torch.full((d.batch, d.n_queries, d.n_heads * d.d_head), float("nan")).pin_memory()
        wd = host.wd[0]
        host.m.step_host(0, x, q, oh, wd[0], wd[1], wd[2], xd, qd, od, chunk * d.chunk_frames, d.chunk_frames,
                         design)
        keep.append((x, q))
        outs.append(oh)
    torch.cuda.synchronize()
    st, flags = host.m.device_status()
    assert st == 0, f"device status {st} flags {flags:#x}"
    for chunk, oh in zip((6, 7), outs):
        dev.append_chunk(0, chunk)
        ref, _ = dev.attend(0, chunk, design=design)
        assert np.array_equal(oh.numpy(), ref), f"chunk {chunk}: host step differs from the device path"


@pytest.mark.parametrize("design", [api.DESIGN_AUTO, api.DESIGN_ABSORBED])
def test_chunk_step_replayed_from_a_cuda_graph(design):
    """One denoising pass of a chunk (append + attention) captured into a CUDA graph from the
    caller's stream and replayed gives the bits of the same calls made eagerly: every launch is
    enqueued on that stream, and reconstruct-once's side stream (the per-head queries) joins the
    capture through its fork and join events.  The eager call comes first, so the handle's stream
    and events exist before the capture."""
    import torch
    d = SMALL
    ro = Rollout(d, design=design)
    _fill(ro, 7)
    chunk = 6
    first = chunk * d.chunk_frames
    x = to_dev(synth.activations(d, 0, chunk, 1), d)
    q = to_dev(synth.queries(d, 0, chunk, 1), d)
    wd = ro.wd[0]
    out_e = torch.full((d.batch, d.n_queries, d.n_heads * d.d_head), float("nan"), dtype=torch.float32,
                       device="cuda")
    out_g = torch.full_like(out_e, float("nan"))
    ro.m.append(0, x, wd[0], first, d.chunk_frames)
    ro.m.attention(0, q, wd[1], wd[2], out_e, first, d.chunk_frames, design)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    cs = torch.cuda.Stream()
    cs.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cs):
        with torch.cuda.graph(g, stream=cs):
            ro.m.append(0, x, wd[0], first, d.chunk_frames)
            ro.m.attention(0, q, wd[1], wd[2], out_g, first, d.chunk_frames, design)
    torch.cuda.synchronize()
    assert torch.isnan(out_g).all(), "capture must not run the kernels"
    g.replay()
    torch.cuda.synchronize()
    st, flags = ro.m.device_status()
    assert st == 0, f"device status {st} flags {flags:#x}"
    assert torch.equal(out_g, out_e), "graph replay differs from the eager calls"
    del g


# ------------------------------------------------------------------ the full Wan-1.3B layer

def test_wan_layer_full_every_design():
    """The Wan-1.3B layer call checked in full: all 4680 query rows x 12 heads over the 32760-key
    window (18 past + 3 current frames, ragged last query tile) against the fp64 oracle, for the
    design AUTO takes there (reconstruct-once), the absorbed design, reconstruct-in-tile and the
    dense per-head cache.  One oracle evaluation serves every design."""
    import time
    ro = Rollout(WAN, design=api.DESIGN_RECON_ONCE, dense=True)
    for c in range(7):
        ro.append_chunk(0, c)
        ro.append_chunk(0, c, dense=True)
    got = {}
    for name, design, dense in (("auto", api.DESIGN_AUTO, False), ("absorbed", api.DESIGN_ABSORBED, False),
                                ("reconstruct_in_tile", api.DESIGN_RECONSTRUCT, False), ("dense", None, True)):
        out, q = ro.attend(0, 6, design=design or api.DESIGN_AUTO, dense=dense)
        got[name] = out[0]
    t0 = time.perf_counter()
    ref = ro.oracle(0, 6, q)
    print(f"oracle, full Wan layer call: {time.perf_counter() - t0:.1f} s")
    for name, o in got.items():
        rel, mx = assert_bf16_close(o, ref, f"wan layer, {name}")
        print(f"wan layer full, {name}: relative L2 {rel:.2e}, max |err| / rms {mx:.2e}")


def test_wan_layer_first_chunk_auto():
    """AUTO on the first chunk of a rollout (3 frames, 4680 keys: reconstruct-once from 4096 keys
    on), 256 seeded query rows of every head."""
    ro = Rollout(WAN)
    _fill(ro, 1)
    out, q = ro.attend(0, 0)
    rows = sampled_rows(WAN.n_queries, 256, seed=3)
    assert_bf16_close(out[0][rows], ro.oracle(0, 0, q, rows=rows), "wan layer, first chunk")


@pytest.mark.parametrize("design", [api.DESIGN_ABSORBED, api.DESIGN_RECON_ONCE])
def test_wide_grid_rotary_pairs_evaluated_directly(design):
    """A 4 x 520 latent grid: the rotary (cos, sin) pairs no longer fit the per-CTA tables (the w
    axis alone has 5 x 520 entries), so the q-absorb kernel (absorbed design) evaluates them per
    query row and the reconstruction (reconstruct-once) per key; two chunks (12480 keys, 6240
    queries), 256 seeded query rows checked for every head."""
    d = SMALL.replace(name="wan_wide_grid", grid_h=4, grid_w=520)
    ro = Rollout(d, design=design)
    _fill(ro, 2)
    out, q = ro.attend(0, 1, design=design)
    rows = sampled_rows(d.n_queries)
    assert_bf16_close(out[0][rows], ro.oracle(0, 1, q, rows=rows), f"wide grid, design {design}")


# ------------------------------------------------------------------ W_uv folded into the output mixer

@pytest.mark.parametrize("d_rope", [32, 16, 64, 96])
def test_small_bf16_folded_output_mixer(d_rope):
    """out = sum_h (W_O,h W_uv,h) o~_h through the library (weight fold, absorbed
    attention handing o~ over as a bf16 pair, one K = 12 x 192 GEMM) against W_O
    applied to the oracle's per-head outputs; every content/rotary split."""
    import torch
    import oracle.vmla_oracle as O
    d = SMALL if d_rope == 32 else split_dims(SMALL, d_rope)
    ro = Rollout(d)
    _fill(ro, 7)
    w = ro.w[0]
    w_fold = torch.empty(d.d_model, d.n_heads * d.d_latent, dtype=torch.bfloat16, device="cuda")
    ro.m.fold_output_weights(to_dev(w.w_o, d), ro.wd[0][2], w_fold)
    ref_fold = O.fold_output_weights(w.w_o, w.w_uv)
    got_fold = w_fold.float().cpu().numpy()
    assert np.all(np.abs(got_fold - ref_fold) <= 2.0 ** -8 * np.abs(ref_fold) + 1e-6 * np.abs(ref_fold).max())
    q = synth.queries(d, 0, 6)
    out = torch.full((1, d.n_queries, d.d_model), float("nan"), dtype=torch.float32, device="cuda")
    ro.m.attention_folded(0, to_dev(q, d), ro.wd[0][1], w_fold, out, 18, 3)
    assert ro.m.device_status()[0] == 0
    heads = ro.oracle(0, 6, q).reshape(d.n_queries, d.n_heads, d.d_head)
    assert_bf16_close(out[0].cpu().numpy(), O.output_projection(heads, w.w_o), "folded output mixer")


# ------------------------------------------------------------------ content path absorbed into the query latent

@pytest.mark.parametrize("d_latent,d_rope", [(128, 32), (192, 32), (192, 16), (192, 64), (128, 96)])
def test_small_bf16_query_latent_absorption(d_latent, d_rope):
    """q~_h = [W_uk,h^T W_uq,h c_Q | RoPE(W_qr,h c_Q)] from the query latent (d_q = 768):
    the library's weight fold and K = 768 query GEMM, then the absorbed attention, against the
    oracle's per-head queries W_uq,h c_Q, W_qr,h c_Q in the non-absorbed definition; the splits
    whose d_latent + d_rope fits one MMA (<= 256)."""
    import torch
    import oracle.vmla_oracle as O
    d = SMALL.replace(d_latent=d_latent) if d_rope == 32 else split_dims(SMALL, d_rope, d_latent)
    ro = Rollout(d)
    _fill(ro, 7)
    w_uq, w_qr = synth.query_latent_weights(d, 0)
    w_qabs = torch.empty(d.n_heads, d.d_latent + d.d_rope, d.d_q, dtype=torch.bfloat16, device="cuda")
    ro.m.fold_query_weights(to_dev(w_uq, d), to_dev(w_qr, d), ro.wd[0][1], w_qabs)
    ref_w = O.fold_query_weights(w_uq, w_qr, ro.w[0].w_uk)
    got_w = w_qabs.float().cpu().numpy()
    assert np.all(np.abs(got_w - ref_w) <= 2.0 ** -8 * np.abs(ref_w) + 1e-6 * np.abs(ref_w).max())
    c_q = synth.query_latents(d, 0, 6)
    out = torch.full((1, d.n_queries, d.n_heads * d.d_head), float("nan"), dtype=torch.float32, device="cuda")
    ro.m.attention_qlatent(0, to_dev(c_q, d), w_qabs, ro.wd[0][2], out, 18, 3)
    assert ro.m.device_status()[0] == 0
    q = O.query_from_latent(c_q[0], w_uq, w_qr)[None]
    assert_bf16_close(out[0].cpu().numpy(), ro.oracle(0, 6, q), f"query latent, d_c={d_latent}")


# ------------------------------------------------------------------ sink frame + local window

def test_tiny_fp32_sink_window():
    """One pinned sink frame and a 3-frame local part, 1-frame chunks: partial
    windows, then every later chunk evicts the oldest local frame only."""
    d = TINY.replace(window_frames=4, sink_frames=1)
    ro = Rollout(d)
    for chunk in range(10):
        ro.append_chunk(0, chunk)
        out, q = ro.attend(0, chunk)
        assert_fp32_close(out[0], ro.oracle(0, chunk, q), f"sink chunk {chunk}")


@pytest.mark.parametrize("design,first", [(api.DESIGN_ABSORBED, 0), (api.DESIGN_RECON_ONCE, 0),
                                          (api.DESIGN_RECONSTRUCT, 1)])
def test_small_bf16_sink_window_rolling(design, first):
    """The long-horizon context of the pages (one sink frame + six recent frames,
    window-relative RoPE) over 9 chunks of 3 frames: the sink stays, the local
    frames rotate, positions stay within 0..6; every chunk checked in full (from the second
    for reconstruct-in-tile, whose first 600-key window is the strict expected failure below)."""
    d = synth.WAN_SMALL_SINK
    ro = Rollout(d, design=api.DESIGN_RECON_ONCE)
    for chunk in range(9):
        ro.append_chunk(0, chunk)
        out, q = ro.attend(0, chunk, design=design)
        if chunk >= first:
            assert_bf16_close(out[0], ro.oracle(0, chunk, q), f"sink chunk {chunk}")


@SHORT_WINDOW_FAILS
def test_small_bf16_sink_window_first_chunk_reconstruct_in_tile():
    d = synth.WAN_SMALL_SINK
    ro = Rollout(d)
    ro.append_chunk(0, 0)
    out, q = ro.attend(0, 0, design=api.DESIGN_RECONSTRUCT)
    assert_bf16_close(out[0], ro.oracle(0, 0, q), "sink chunk 0, reconstruct-in-tile")


def test_small_bf16_sink_window_passes_and_noalloc():
    """Two denoising passes per chunk on the sink window (absorbed design), then the allocation-free
    entry point on the same window: equal bit for bit."""
    import torch
    d = synth.WAN_SMALL_SINK
    ro = Rollout(d)
    for chunk in range(5):
        for p in range(2):
            ro.append_chunk(0, chunk, pass_=p)
            out, q = ro.attend(0, chunk, pass_=p, design=api.DESIGN_ABSORBED)
            assert_bf16_close(out[0], ro.oracle(0, chunk, q), f"sink chunk {chunk} pass {p}")
    qd = to_dev(q, d)
    out2 = torch.empty_like(torch.from_numpy(out)).cuda()
    api.check(api.lib().vmla_chunk_attention_noalloc(ro.cfg, 0, ro.m.ckv.data_ptr(), ro.m.kr.data_ptr(), 15,
                                                     qd.data_ptr(), ro.wd[0][1].data_ptr(), ro.wd[0][2].data_ptr(),
                                                     out2.data_ptr(), 12, 3, torch.cuda.current_stream().cuda_stream),
              "noalloc")
    assert ro.m.device_status()[0] == 0
    assert torch.equal(out2.cpu(), torch.from_numpy(out)), "allocation-free path differs on the sink window"


@pytest.mark.parametrize("chunk,pass_", [(0, 0), pytest.param(0, 1, marks=pytest.mark.xfail(
    strict=True, reason="fails the max-error gate at the bf16 cache's own floor: on this 600-key window the "
                        "cache rounding alone gives 2.8e-2 RMS (fp64 emulation), reconstruct-once 3.08e-2")),
    (1, 1), (4, 1)])
def test_small_bf16_sink_window_passes_reconstruct_once(chunk, pass_):
    """Reconstruct-once (AUTO at d_latent 192) on the sink window's denoising passes."""
    d = synth.WAN_SMALL_SINK
    ro = Rollout(d)
    for c in range(chunk + 1):
        for p in range(2 if c < chunk else pass_ + 1):
            ro.append_chunk(0, c, pass_=p)
    out, q = ro.attend(0, chunk, pass_=pass_, design=api.DESIGN_RECON_ONCE)
    assert_bf16_close(out[0], ro.oracle(0, chunk, q), f"sink chunk {chunk} pass {pass_}, reconstruct-once")


# ------------------------------------------------------------------ numerics of the kernels' helpers

def test_polynomial_exp2_error_bound():
    """The FMA-pipe 2^x of the softmax loops against fp64 exp2: relative error
    within the fitted minimax bound (7.5e-5) for x >= -125, tiny below."""
    import torch
    x = np.concatenate([np.linspace(-125.0, 10.0, 1 << 20), np.linspace(-0.5, 0.5, 4096),
                        np.arange(-125, 11, dtype=np.float64) + 0.5, [-126.0, -200.0, -1e30, -np.inf]])
    x = x[: len(x) // 2 * 2].astype(np.float32)
    xd = torch.from_numpy(x).cuda()
    yd = torch.empty_like(xd)
    api.selftest_exp2(xd, yd)
    y = yd.cpu().numpy().astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    ok = x >= -125
    rel = np.abs(y[ok] - ref[ok]) / ref[ok]
    assert rel.max() <= 7.6e-5, rel.max()
    assert np.all(np.isfinite(y)) and np.all(y[~ok] >= 0) and np.all(y[~ok] <= 2.0 ** -124)


# ------------------------------------------------------------------ failure detection

def test_bounded_wait_times_out_and_reports():
    import torch
    api.selftest_wait_timeout(20_000_000)
    m = api.LatentKVAttention(api.config_from_dims(TINY))
    st, flags = m.device_status()
    assert st == 5 and flags & 16
    assert m.device_status()[0] == 0  # cleared
    torch.cuda.synchronize()
