"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each ``check_*`` takes the oracle module (or a mutant of it) and raises
AssertionError when the oracle disagrees with its pin.  The tests run every
check on the oracle itself, then plant plausible mistakes in copies of the
oracle (on the CPU) and require that some check catches each one.
"""
import collections
import math
import types

import numpy as np
import pytest
import torch

import oracle.vmla_oracle as O
from latent_kv_attention_down_b200 import synth

RNG = np.random.default_rng(1234)


def _rand(*shape, rng=RNG):
    return rng.standard_normal(shape)


def _tiny_scenario(orc, dims=synth.TINY, frames_appended=None, seed=0, rope_at="read", n_keys_frames=None):
    """A window of the tiny layer filled from seeded x, and one chunk of queries."""
    d = dims
    wts = synth.weights(d, layer=0, base_seed=seed)
    F = d.window_frames if frames_appended is None else frames_appended
    frame_x = {f: synth.activations(d, 0, f, n_frames=1, base_seed=seed)[0] for f in range(F)}
    c, r, kpos, t0 = orc.window_latents(frame_x, F, d.window_frames, wts.w_down, d.d_latent,
                                        d.grid_h, d.grid_w, rope_at=rope_at)
    first = F - d.chunk_frames
    q = synth.queries(d, 0, first, base_seed=seed)[0]
    qpos = orc.chunk_query_positions(first, d.chunk_frames, t0, d.grid_h, d.grid_w)
    return c, r, kpos, q, qpos, wts


KW = dict(d_nope=synth.TINY.d_nope, rope_pairs=synth.TINY.rope_pairs)


# ---------------------------------------------------------------- page numbers

def check_page_numbers(orc, golden):
    g = {k: v["value"] for k, v in golden.items()}
    lat = orc.latent_scalars_per_token(g["d_latent"], g["d_rope"])
    den = orc.dense_scalars_per_token(g["n_heads"], g["d_head"])
    assert lat == g["latent_scalars_per_token"]
    assert den == g["dense_scalars_per_token"]
    assert round(100.0 * (1 - lat / den), 1) == g["reduction_percent"]
    assert round(den / lat, 1) == g["reduction_ratio"]
    assert g["latent_frames_per_clip"] * g["tokens_per_latent_frame"] == g["tokens_per_clip"]
    dense = orc.cache_scalars(g["latent_frames_per_clip"], g["tokens_per_latent_frame"], g["layers"], den)
    assert round(dense / 1e9, 2) == g["dense_cache_scalars_billion"]
    assert round(dense * 2 / 1e9, 1) == g["dense_cache_gb_bf16"]
    assert 2 * sum(g["rope_pairs_thw"]) == g["d_rope"]
    assert sum(g["nope_rope_split"]) == g["d_head"] and g["nope_rope_split"][1] == g["d_rope"]
    assert orc.ROPE_MAX_POSITION == g["rope_max_length_per_axis"]


def test_page_numbers(golden):
    check_page_numbers(O, golden)


# ---------------------------------------------------------------- RoPE

def check_rope_frequencies(orc):
    f = orc.rope_frequencies((6, 5, 5), 10000.0)
    assert [len(a) for a in f] == [6, 5, 5]
    # highest band of every axis turns at 1 rad per position
    assert all(a[0] == 1.0 for a in f)
    # closed forms: 10000^(-2*3/12) = 1/100, 10000^(-2/12) = 10^(-2/3), 10000^(-2*4/10) = 10^(-16/5)
    np.testing.assert_allclose(f[0][3], 0.01, rtol=1e-15)
    np.testing.assert_allclose(f[0][1], 0.21544346900318834, rtol=1e-15)
    np.testing.assert_allclose(f[1][4], 6.309573444801929e-04, rtol=1e-14)
    np.testing.assert_allclose(f[2][4], 6.309573444801929e-04, rtol=1e-14)
    # strictly decreasing
    assert all(np.all(np.diff(a) < 0) for a in f)
    # a larger per-axis band group: the highest-frequency n_a bands of it
    g = orc.rope_frequencies((6, 5, 5), 10000.0, (44, 42, 42))
    np.testing.assert_allclose(g[0][1], 10000.0 ** (-1 / 22), rtol=1e-15)
    np.testing.assert_allclose(g[1][2], 10000.0 ** (-2 / 21), rtol=1e-15)


def check_rope_complex(orc):
    """Pair rotation = multiplication of (v[2i] + i v[2i+1]) by exp(i*angle)."""
    v = _rand(7, 32)
    ang = _rand(7, 16) * 5
    got = orc.rope_rotate(v, ang)
    z = (v[:, 0::2] + 1j * v[:, 1::2]) * np.exp(1j * ang)
    np.testing.assert_allclose(got[:, 0::2], z.real, atol=1e-14)
    np.testing.assert_allclose(got[:, 1::2], z.imag, atol=1e-14)


def check_rope_norm_and_identity(orc):
    f = orc.rope_frequencies((6, 5, 5))
    v = _rand(50, 32)
    pos = RNG.integers(0, 1024, size=(50, 3))
    ang = orc.rope_angles(pos[:, 0], pos[:, 1], pos[:, 2], f)
    rv = orc.rope_rotate(v, ang)
    np.testing.assert_allclose(np.linalg.norm(rv, axis=1), np.linalg.norm(v, axis=1), rtol=1e-14)
    z = orc.rope_rotate(v, orc.rope_angles(0 * pos[:, 0], 0 * pos[:, 1], 0 * pos[:, 2], f))
    np.testing.assert_array_equal(z, v)


def check_rope_relative(orc):
    """q.k after rotation depends only on the (t, h, w) offset: shifting both
    positions by the same amount on any axis leaves every score unchanged,
    shifting one of them does not."""
    f = orc.rope_frequencies((6, 5, 5))
    a, b = _rand(40, 32), _rand(40, 32)
    p1 = RNG.integers(0, 60, size=(40, 3))
    p2 = RNG.integers(0, 60, size=(40, 3))

    def score(pa, pb):
        ra = orc.rope_rotate(a, orc.rope_angles(pa[:, 0], pa[:, 1], pa[:, 2], f))
        rb = orc.rope_rotate(b, orc.rope_angles(pb[:, 0], pb[:, 1], pb[:, 2], f))
        return np.sum(ra * rb, axis=1)

    s0 = score(p1, p2)
    for axis in range(3):
        d = np.zeros(3, dtype=np.int64)
        d[axis] = 17
        np.testing.assert_allclose(score(p1 + d, p2 + d), s0, atol=1e-11)
        assert np.max(np.abs(score(p1 + d, p2) - s0)) > 1e-3


def check_rope_axis_layout(orc):
    """t turns the first 2*6 dims, h the next 2*5, w the last 2*5."""
    f = orc.rope_frequencies((6, 5, 5))
    v = _rand(3, 32)
    base = orc.rope_rotate(v, orc.rope_angles(np.zeros(3), np.zeros(3), np.zeros(3), f))
    spans = {0: slice(0, 12), 1: slice(12, 22), 2: slice(22, 32)}
    for axis in range(3):
        pos = [np.zeros(3)] * 3
        pos = [p.copy() for p in pos]
        pos[axis] = np.full(3, 5.0)
        rv = orc.rope_rotate(v, orc.rope_angles(*pos, f))
        moved = np.any(np.abs(rv - base) > 1e-12, axis=0)
        expect = np.zeros(32, dtype=bool)
        expect[spans[axis]] = True
        assert np.array_equal(moved, expect), (axis, moved)


@pytest.mark.parametrize("check", [check_rope_frequencies, check_rope_complex, check_rope_norm_and_identity,
                                   check_rope_relative, check_rope_axis_layout])
def test_rope(check):
    check(O)


@pytest.mark.parametrize("pairs", [(4, 2, 2), (12, 10, 10), (16, 16, 16)])
def test_rope_other_rotary_splits(pairs):
    """The 16, 64 and 96 rotary-dim layouts: every axis's first band turns at 1 rad per position
    and, with the default base 2*n_a, band n_a/2 at 10000^(-1/2) = 0.01; each axis turns its own
    2*n_a dims, in t, h, w order; scores stay invariant under a common shift on any axis and move
    under a one-sided one."""
    f = O.rope_frequencies(pairs)
    assert [len(a) for a in f] == list(pairs)
    for a, n in zip(f, pairs):
        assert a[0] == 1.0
        np.testing.assert_allclose(a[n // 2], 0.01, rtol=1e-14)
        assert np.all(np.diff(a) < 0)
    dr = 2 * sum(pairs)
    v = _rand(3, dr)
    zero = np.zeros(3)
    base = O.rope_rotate(v, O.rope_angles(zero, zero, zero, f))
    edges = np.cumsum([0] + [2 * n for n in pairs])
    for axis in range(3):
        pos = [zero.copy() for _ in range(3)]
        pos[axis] = np.full(3, 5.0)
        moved = np.any(np.abs(O.rope_rotate(v, O.rope_angles(*pos, f)) - base) > 1e-12, axis=0)
        expect = np.zeros(dr, dtype=bool)
        expect[edges[axis]:edges[axis + 1]] = True
        assert np.array_equal(moved, expect), (pairs, axis)
    a_, b_ = _rand(30, dr), _rand(30, dr)
    p1, p2 = RNG.integers(0, 60, size=(30, 3)), RNG.integers(0, 60, size=(30, 3))

    def score(pa, pb):
        ra = O.rope_rotate(a_, O.rope_angles(pa[:, 0], pa[:, 1], pa[:, 2], f))
        rb = O.rope_rotate(b_, O.rope_angles(pb[:, 0], pb[:, 1], pb[:, 2], f))
        return np.sum(ra * rb, axis=1)

    s0 = score(p1, p2)
    for axis in range(3):
        d = np.zeros(3, dtype=np.int64)
        d[axis] = 23
        np.testing.assert_allclose(score(p1 + d, p2 + d), s0, atol=1e-11)
        assert np.max(np.abs(score(p1 + d, p2) - s0)) > 1e-3


# ---------------------------------------------------------------- ring / window

def check_ring_against_deque(orc, W=21, chunk=3, chunks=20):
    """FIFO window = a deque of maxlen W; ring slots never overwrite a frame
    that is still in the window, and every window frame is where it was put."""
    dq = collections.deque(maxlen=W)
    ring = [None] * W
    F = 0
    for _ in range(chunks):
        for f in range(F, F + chunk):
            dq.append(f)
            ring[orc.ring_slot(f, W)] = f
        F += chunk
        start, end = orc.window_frame_range(F, W)
        assert list(range(start, end)) == list(dq)
        for f in dq:
            assert ring[orc.ring_slot(f, W)] == f
        assert sorted(orc.ring_slot(f, W) for f in dq) == sorted(set(orc.ring_slot(f, W) for f in dq))


def test_ring():
    check_ring_against_deque(O)
    check_ring_against_deque(O, W=4, chunk=1, chunks=9)
    check_ring_against_deque(O, W=7, chunk=2, chunks=11)  # chunks straddle the wrap


def test_token_positions():
    h, w = O.token_grid_position(np.arange(1560), 52)
    assert h.max() == 29 and w.max() == 51
    assert h[52] == 1 and w[52] == 0 and h[51] == 0 and w[51] == 51
    kp = O.key_positions([5, 6], 5, 30, 52)
    assert kp.shape == (3120, 3) and kp[0].tolist() == [0, 0, 0] and kp[-1].tolist() == [1, 29, 51]


# ---------------------------------------------------------------- attention

def check_softmax_vs_sdpa(orc):
    q, k, v = _rand(9, 16), _rand(33, 16), _rand(33, 5)
    got = orc.softmax_attention(q, k, v, 1 / math.sqrt(16))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None]).numpy()[0]
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)


def check_chunk_vs_sdpa(orc):
    """The whole chunk attention against torch's attention routine on keys and
    values rebuilt head by head (q rotated by the same positions)."""
    c, r, kpos, q, qpos, wts = _tiny_scenario(orc)
    got = orc.chunk_attention(c, r, kpos, q, qpos, wts.w_uk, wts.w_uv, **KW)
    k, v = orc.dense_cache_entries(c, r, kpos, wts.w_uk, wts.w_uv, rope_pairs=KW["rope_pairs"])
    qr = orc.rotate_queries(q, qpos, KW["d_nope"], orc.rope_frequencies(KW["rope_pairs"]))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(qr).transpose(0, 1), torch.from_numpy(k).transpose(0, 1),
        torch.from_numpy(v).transpose(0, 1)).transpose(0, 1).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)


def check_absorbed_equals_reconstructed(orc, dims=synth.TINY):
    c, r, kpos, q, qpos, wts = _tiny_scenario(orc, dims)
    kw = dict(d_nope=dims.d_nope, rope_pairs=dims.rope_pairs)
    a = orc.chunk_attention(c, r, kpos, q, qpos, wts.w_uk, wts.w_uv, **kw)
    b = orc.chunk_attention_absorbed(c, r, kpos, q, qpos, wts.w_uk, wts.w_uv, **kw)
    np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-12)


def check_single_key(orc):
    """One key: every query returns that key's value, v_h = W_uv,h c."""
    c, r, kpos, q, qpos, wts = _tiny_scenario(orc)
    out = orc.chunk_attention(c[:1], r[:1], kpos[:1], q, qpos, wts.w_uk, wts.w_uv, **KW)
    expect = np.stack([wts.w_uv[h].astype(np.float64) @ c[0] for h in range(2)])
    np.testing.assert_allclose(out, np.broadcast_to(expect, out.shape), rtol=1e-12, atol=1e-13)


def check_zero_query(orc):
    """q = 0: uniform weights, so the output is the mean value over the window."""
    c, r, kpos, q, qpos, wts = _tiny_scenario(orc)
    out = orc.chunk_attention(c, r, kpos, 0 * q, qpos, wts.w_uk, wts.w_uv, **KW)
    mean_c = c.mean(axis=0)
    expect = np.stack([wts.w_uv[h].astype(np.float64) @ mean_c for h in range(2)])
    np.testing.assert_allclose(out, np.broadcast_to(expect, out.shape), rtol=1e-12, atol=1e-13)


def check_key_permutation(orc):
    c, r, kpos, q, qpos, wts = _tiny_scenario(orc)
    perm = np.random.default_rng(7).permutation(c.shape[0])
    a = orc.chunk_attention(c, r, kpos, q, qpos, wts.w_uk, wts.w_uv, **KW)
    b = orc.chunk_attention(c[perm], r[perm], kpos[perm], q, qpos, wts.w_uk, wts.w_uv, **KW)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)


def check_single_head_no_rope(orc):
    """n_h = 1 and no positional dims: plain softmax attention with k = W_uk c, v = W_uv c."""
    d = synth.TINY.replace(n_heads=1, d_rope=0, rope_pairs=(0, 0, 0))
    c, r, kpos, q, qpos, wts = _tiny_scenario(orc, d)
    out = orc.chunk_attention(c, r, kpos, q, qpos, wts.w_uk, wts.w_uv, d_nope=d.d_nope, rope_pairs=(0, 0, 0))
    k = c @ wts.w_uk[0].astype(np.float64).T
    v = c @ wts.w_uv[0].astype(np.float64).T
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q[:, 0].astype(np.float64))[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None])
    np.testing.assert_allclose(out[:, 0], ref.numpy()[0], rtol=1e-12, atol=1e-13)


def check_brute_force(orc):
    """Loop-by-loop evaluation of the definition on the tiny case."""
    d = synth.TINY
    c, r, kpos, q, qpos, wts = _tiny_scenario(orc)
    got = orc.chunk_attention(c, r, kpos, q, qpos, wts.w_uk, wts.w_uv, **KW)
    om = [1.0, 1.0, 1.0]  # one pair per axis: theta^0

    def rot(vec, pos):
        out = list(vec)
        for i in range(3):
            a = pos[i] * om[i]
            u, w = vec[2 * i], vec[2 * i + 1]
            out[2 * i] = u * math.cos(a) - w * math.sin(a)
            out[2 * i + 1] = u * math.sin(a) + w * math.cos(a)
        return out

    for h in range(d.n_heads):
        keys, vals = [], []
        for j in range(c.shape[0]):
            kn = [sum(float(wts.w_uk[h, e, m]) * c[j, m] for m in range(d.d_latent)) for e in range(d.d_nope)]
            keys.append(kn + rot(list(r[j]), kpos[j]))
            vals.append([sum(float(wts.w_uv[h, e, m]) * c[j, m] for m in range(d.d_latent)) for e in range(d.d_head)])
        for i in range(q.shape[0]):
            qq = [float(v) for v in q[i, h, :d.d_nope]] + rot([float(v) for v in q[i, h, d.d_nope:]], qpos[i])
            s = [sum(a * b for a, b in zip(qq, kk)) / math.sqrt(d.d_head) for kk in keys]
            m = max(s)
            e = [math.exp(x - m) for x in s]
            z = sum(e)
            o = [sum(e[j] * vals[j][t] for j in range(len(keys))) / z for t in range(d.d_head)]
            np.testing.assert_allclose(got[i, h], o, rtol=1e-11, atol=1e-12)


def check_read_equals_append(orc):
    """Window-relative and absolute frame numbering give the same attention
    (RoPE depends on offsets only) -- the cache is independent of absolute
    rollout time."""
    d = synth.TINY
    a = _tiny_scenario(orc, d, frames_appended=9, rope_at="read")
    b = _tiny_scenario(orc, d, frames_appended=9, rope_at="append")
    assert a[2][0, 0] == 0 and b[2][0, 0] == 5
    oa = orc.chunk_attention(*a[:5], a[5].w_uk, a[5].w_uv, **KW)
    ob = orc.chunk_attention(*b[:5], b[5].w_uk, b[5].w_uv, **KW)
    np.testing.assert_allclose(oa, ob, rtol=1e-11, atol=1e-12)


ATTN_CHECKS = [check_softmax_vs_sdpa, check_chunk_vs_sdpa, check_absorbed_equals_reconstructed, check_single_key,
               check_zero_query, check_key_permutation, check_single_head_no_rope, check_brute_force,
               check_read_equals_append]


@pytest.mark.parametrize("check", ATTN_CHECKS)
def test_attention(check):
    check(O)


def test_absorbed_equals_reconstructed_wan_dims():
    d = synth.WAN.replace(name="wan_pin", grid_h=3, grid_w=4, window_frames=5, chunk_frames=2)
    check_absorbed_equals_reconstructed(O, d)


# ---------------------------------------------------------------- planted mistakes

def _mutant(**overrides):
    m = types.ModuleType("mutant")
    m.__dict__.update({k: v for k, v in O.__dict__.items() if not k.startswith("__")})
    m.__dict__.update(overrides)
    # functions keep the real module as their globals; rebind them so the
    # overrides are seen by every caller inside the mutant
    for k, v in list(m.__dict__.items()):
        if isinstance(v, types.FunctionType) and k not in overrides:
            m.__dict__[k] = types.FunctionType(v.__code__, m.__dict__, k, v.__defaults__, v.__closure__)
            m.__dict__[k].__kwdefaults__ = v.__kwdefaults__
    return m


def _rope_sign_flip(v, angles):
    return O.rope_rotate(v, -np.asarray(angles))


def _rope_axis_swap(t, h, w, freqs):
    return O.rope_angles(h, t, w, [freqs[1], freqs[0], freqs[2]]) if len(freqs[0]) == len(freqs[1]) \
        else O.rope_angles(w, h, t, freqs)


def _freq_wrong_base(pairs, theta=10000.0, base_dims=None):
    return [np.power(float(theta), -np.arange(n) / float(max(n, 1))) for n in pairs]


def _softmax_no_max(q, k, v, scale):
    s = (q @ k.T) * (1.0 / math.sqrt(q.shape[1] - 1))
    p = np.exp(s)
    return (p / p.sum(axis=1, keepdims=True)) @ v


def _window_off_by_one(frames_appended, window_frames):
    return max(0, frames_appended - window_frames + 1), frames_appended


def _reconstruct_no_rope(c, k_rope, w_uk, w_uv):
    k, v = O.reconstruct_heads(c, 0 * k_rope, w_uk, w_uv)
    return k, v


def _sink_local_t_from_zero(frames_appended, window_frames, sink_frames=0):
    frames = O.window_frames_list(frames_appended, window_frames, sink_frames)
    return {f: (k if k < sink_frames else k - sink_frames) for k, f in enumerate(frames)}


def _sink_evicted(frames_appended, window_frames, sink_frames=0):
    return O.window_frames_list(frames_appended, window_frames, 0)


MUTANTS = {
    "rope rotates the wrong way": dict(rope_rotate=_rope_sign_flip),
    "rope axes in the wrong order": dict(rope_angles=_rope_axis_swap),
    "rope band base wrong": dict(rope_frequencies=_freq_wrong_base),
    "softmax scale wrong": dict(softmax_attention=_softmax_no_max),
    "window one frame short": dict(window_frame_range=_window_off_by_one),
    "positional score dropped from the per-head keys": dict(reconstruct_heads=_reconstruct_no_rope),
    "sink window: local frames counted from t = 0": dict(window_frame_t=_sink_local_t_from_zero),
    "sink window: the sink frame evicted like the others": dict(window_frames_list=_sink_evicted),
}


def _all_checks(orc, golden):
    check_page_numbers(orc, golden)
    for chk in (check_rope_frequencies, check_rope_complex, check_rope_norm_and_identity, check_rope_relative,
                check_rope_axis_layout, check_ring_against_deque):
        chk(orc)
    for chk in ATTN_CHECKS:
        chk(orc)
    check_sink_slot_array(orc)
    check_sink_attention_brute_force(orc)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, golden):
    with pytest.raises(AssertionError):
        _all_checks(_mutant(**MUTANTS[name]), golden)


def test_unmutated_passes_all(golden):
    _all_checks(_mutant(), golden)


# ---------------------------------------------------------------- sink frame + local window
def _simulate_sink_ring(n_frames, W, S):
    """An explicit slot array: sink frames take their own slot; a later frame takes
    the first never-used local slot, else the slot of the oldest local frame."""
    slots = [None] * W
    states = []
    for f in range(n_frames):
        if f < S:
            s = f
        else:
            free = [k for k in range(S, W) if slots[k] is None]
            s = free[0] if free else min(range(S, W), key=lambda k: slots[k])
        slots[s] = f
        states.append(list(slots))
    return states


def check_sink_slot_array(orc, W=7, S=1):
    states = _simulate_sink_ring(60, W, S)
    for F in range(1, 61):
        slots = states[F - 1]
        frames = orc.window_frames_list(F, W, S)
        assert sorted(frames) == sorted(f for f in slots if f is not None)
        for k, f in enumerate(slots):
            if f is not None:
                assert orc.ring_slot(f, W, S) == k
        # sink first, locals oldest first, window-relative t = position in that order
        t = orc.window_frame_t(F, W, S)
        sink = [f for f in frames if f < S]
        local = [f for f in frames if f >= S]
        assert frames == sink + sorted(local)
        assert [t[f] for f in frames] == list(range(len(frames)))
        if S == 0:
            assert frames == list(range(*orc.window_frame_range(F, W)))


@pytest.mark.parametrize("W,S", [(7, 1), (4, 1), (5, 2), (21, 0)])
def test_sink_window_matches_an_explicit_slot_array(W, S):
    check_sink_slot_array(O, W, S)


def test_sink_window_keeps_rope_positions_bounded():
    """One sink frame and a six-frame local window [paperlayer App. D.4, D.5]: after
    1000 frames the temporal coordinates are still 0..6 and the sink is frame 0."""
    frames = O.window_frames_list(1000, 7, 1)
    t = O.window_frame_t(1000, 7, 1)
    assert frames == [0] + list(range(994, 1000))
    assert sorted(t.values()) == list(range(7)) and t[0] == 0 and t[999] == 6


def test_sink_window_latents_positions():
    rng = np.random.default_rng(3)
    T, D, dc = 6, 8, 4
    frame_x = {f: rng.standard_normal((T, D)) for f in range(12)}
    w = rng.standard_normal((dc + 2, D))
    c, r, pos, t0 = O.window_latents(frame_x, 12, 4, w, dc, 2, 3, sink_frames=1)
    assert c.shape == (4 * T, dc)
    np.testing.assert_allclose(c[:T], frame_x[0] @ w[:dc].T)     # the sink's rows come first
    np.testing.assert_allclose(c[T:2 * T], frame_x[9] @ w[:dc].T)
    assert list(pos[::T, 0]) == [0, 1, 2, 3] and t0 == 8         # frames 9, 10, 11 at t = 1, 2, 3
    q = O.chunk_query_positions(11, 1, t0, 2, 3)
    assert q[0, 0] == 3


# ---------------------------------------------------------------- output mixer folded into the value path
def test_folded_output_equals_projected_heads():
    """sum_h (W_O,h W_uv,h) o~_h (absorbed all the way into the output mixer) equals
    W_O applied to the concatenated per-head outputs of the non-absorbed definition."""
    rng = np.random.default_rng(11)
    n_h, d_nope, d_rope, d_c, N_k, N_q, d_out = 3, 6, 4, 5, 17, 7, 9
    c = rng.standard_normal((N_k, d_c))
    r = rng.standard_normal((N_k, d_rope))
    kpos = rng.integers(0, 6, (N_k, 3))
    q = rng.standard_normal((N_q, n_h, d_nope + d_rope))
    qpos = rng.integers(0, 6, (N_q, 3))
    w_uk = rng.standard_normal((n_h, d_nope, d_c))
    w_uv = rng.standard_normal((n_h, d_nope + d_rope, d_c))
    w_o = rng.standard_normal((d_out, n_h * (d_nope + d_rope)))
    kw = dict(d_nope=d_nope, rope_pairs=(1, 0, 1))
    ref = O.output_projection(O.chunk_attention(c, r, kpos, q, qpos, w_uk, w_uv, **kw), w_o)
    fold = O.fold_output_weights(w_o, w_uv)
    assert fold.shape == (d_out, n_h * d_c)
    got = O.chunk_attention_folded(c, r, kpos, q, qpos, w_uk, fold, **kw)
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)
    # a head block in the wrong place must not pass
    bad = np.concatenate([fold[:, d_c:2 * d_c], fold[:, :d_c], fold[:, 2 * d_c:]], axis=1)
    assert np.abs(O.chunk_attention_folded(c, r, kpos, q, qpos, w_uk, bad, **kw) - ref).max() > 1e-3


# ---------------------------------------------------------------- content path absorbed into the query latent
def test_query_latent_absorption_equals_the_definition():
    """q~_h = [W_uk,h^T W_uq,h c_Q | RoPE(W_qr,h c_Q)] against the shared latent key gives
    what the per-head queries W_uq,h c_Q, W_qr,h c_Q give in the non-absorbed definition."""
    rng = np.random.default_rng(12)
    n_h, d_nope, d_rope, d_c, d_q, N_k, N_q = 2, 6, 4, 5, 11, 13, 6
    c = rng.standard_normal((N_k, d_c))
    r = rng.standard_normal((N_k, d_rope))
    kpos = rng.integers(0, 5, (N_k, 3))
    cq = rng.standard_normal((N_q, d_q))
    qpos = rng.integers(0, 5, (N_q, 3))
    w_uq = rng.standard_normal((n_h, d_nope, d_q))
    w_qr = rng.standard_normal((n_h, d_rope, d_q))
    w_uk = rng.standard_normal((n_h, d_nope, d_c))
    w_uv = rng.standard_normal((n_h, d_nope + d_rope, d_c))
    kw = dict(rope_pairs=(1, 0, 1))
    q = O.query_from_latent(cq, w_uq, w_qr)
    assert q.shape == (N_q, n_h, d_nope + d_rope)
    ref = O.chunk_attention(c, r, kpos, q, qpos, w_uk, w_uv, d_nope=d_nope, **kw)
    w_qabs = O.fold_query_weights(w_uq, w_qr, w_uk)
    assert w_qabs.shape == (n_h, d_c + d_rope, d_q)
    got = O.chunk_attention_query_latent(c, r, kpos, cq, qpos, w_qabs, w_uv, d_latent=d_c, d_head=d_nope + d_rope, **kw)
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)
    bad = w_qabs.copy()
    bad[:, :d_c] = np.einsum("hnc,hnj->hcj", w_uk, w_uq[::-1])   # heads crossed
    assert np.abs(O.chunk_attention_query_latent(c, r, kpos, cq, qpos, bad, w_uv, d_latent=d_c,
                                                 d_head=d_nope + d_rope, **kw) - ref).max() > 1e-3


def check_sink_attention_brute_force(orc):
    """One sink frame and a three-frame local part (W = 4) after ten one-frame chunks, by explicit
    loops: the context is frames 0, 7, 8, 9 at t = 0, 1, 2, 3; every key k_jh = [W_uk,h c_j |
    R(t_j, h_j, w_j) k_R,j] and query [q_nope | R(3, h_i, w_i) q_rope] is rotated pair by pair as a
    complex number, the softmax is taken over the 24 keys one score at a time, and v_jh = W_uv,h c_j.
    The oracle's window, positions and attention must give the same output."""
    rng = np.random.default_rng(21)
    D, n_h, d_nope, d_c, gh, gw, W, S = 5, 2, 4, 3, 2, 3, 4, 1
    pairs = (1, 0, 1)                                 # d_rope = 4: one t pair, one w pair
    d_rope = 2 * sum(pairs)
    T = gh * gw
    w_down = rng.standard_normal((d_c + d_rope, D))
    w_uk = rng.standard_normal((n_h, d_nope, d_c))
    w_uv = rng.standard_normal((n_h, d_nope + d_rope, d_c))
    frame_x = {f: rng.standard_normal((T, D)) for f in range(10)}
    q = rng.standard_normal((T, n_h, d_nope + d_rope))
    # the oracle
    c, r, kpos, t0 = orc.window_latents(frame_x, 10, W, w_down, d_c, gh, gw, sink_frames=S)
    qpos = orc.chunk_query_positions(9, 1, t0, gh, gw)
    got = orc.chunk_attention(c, r, kpos, q, qpos, w_uk, w_uv, d_nope=d_nope, rope_pairs=pairs).reshape(T, n_h, -1)
    # brute force: base 2*n_a gives the single band of an axis a frequency of 1
    context = [(0, 0), (7, 1), (8, 2), (9, 3)]          # (frame, window-relative t)

    def rotate(v, t, hh, ww):                          # v: [t pair | w pair]
        out = np.array(v, dtype=np.float64)
        for k, p in ((0, t), (1, ww)):
            z = complex(v[2 * k], v[2 * k + 1]) * np.exp(1j * p * 1.0)
            out[2 * k], out[2 * k + 1] = z.real, z.imag
        return out

    scale = 1.0 / np.sqrt(d_nope + d_rope)
    for i in range(T):
        hi, wi = divmod(i, gw)
        for h in range(n_h):
            qv = np.concatenate([q[i, h, :d_nope], rotate(q[i, h, d_nope:], 3, hi, wi)])
            scores, values = [], []
            for f, t in context:
                for j in range(T):
                    hj, wj = divmod(j, gw)
                    cj = w_down[:d_c] @ frame_x[f][j]
                    kr = w_down[d_c:] @ frame_x[f][j]
                    k = np.concatenate([w_uk[h] @ cj, rotate(kr, t, hj, wj)])
                    scores.append(float(qv @ k) * scale)
                    values.append(w_uv[h] @ cj)
            m = max(scores)
            e = [np.exp(s - m) for s in scores]
            ref = sum(ei * v for ei, v in zip(e, values)) / sum(e)
            np.testing.assert_allclose(got[i, h], ref, rtol=1e-11, atol=1e-12)


def test_sink_window_attention_brute_force():
    check_sink_attention_brute_force(O)
