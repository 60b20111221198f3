"""Stage-by-stage parity: every kernel of the chunk path against the fp64 definition of its own
step, fed the GPU's stored inputs of that step, so that the rounding of one stage never hides a
defect in the next.

The end-to-end tests compare against the oracle computed from x; there the bf16 rounding of the
224-scalar cache alone uses up to two thirds of the max-error budget.  Here:

* window RoPE: the stored bf16 k_R of the ring, rotated in fp64 at the window-relative positions
  vmla_window reports, against the rotated keys the kernel left in the workspace (bf16 for the
  absorbed design, fp16 for reconstruct-once);
* q-absorb: [W_uk,h^T q_nope | RoPE(q_rope)] in fp64 against the absorbed queries in the workspace;
* per-head queries: [q_nope | RoPE(q_rope)] (the content part must be copied bit for bit);
* reconstruction: [W_uk,h c | k_R rotated] and W_uv,h c from the stored cache against the per-head
  K/V in the workspace (the positional columns must be copied bit for bit);
* attention cores: the textbook softmax attention in fp64 over the GPU's own queries, keys and
  values (absorbed: q~ against [c | k_R rotated], values c, then W_uv; per-head: q_h against K_h,
  values V_h) against the kernel's fp32 output.

Bounds.  One bf16 rounding (round to nearest even, unit roundoff u = 2^-8) of a result r moves
it by at most u |r|; fp32 sums of products add at most a few 2^-24 of the sum of |terms|.  Inside
an attention core the only rounding left is that of the probabilities P to bf16 before P V (the
row sums use the unrounded values; the softmax-weighted latents reach W_uv as a bf16 pair, whose
residual is below 2^-16).  With delta_j the relative rounding of p_j (|delta_j| <= u, independent
across keys, variance u^2 / 3), the error of output element e is sum_j (p_j / l) delta_j v_je, a sum
of independent terms of standard deviation
    sigma_e = u / sqrt(3) * sqrt(sum_j (p_j / l)^2 v_je^2).
The test holds every element to 6 sigma_e plus 1e-4 of RMS(out) for the fp32 arithmetic (score
sums, exp2, the tensor core's accumulation): a Gaussian error passes 6 sigma with probability
2e-9 per element, so over the few million elements checked a correct kernel fails with
probability below 1e-2, while a wrong key, a dropped scale, a wrong rotary angle or a missed
rescale moves elements by tens of sigma.

Where a stage's input is itself the result of two roundings (the dense cache: c = bf16(W_dkv x),
then each entry rounded again), the bound adds u times the sum of |terms| for the inner one.

The reconstruct-once workspace holds the per-head queries, keys and values in fp16, and its
attention core rounds P to fp16: unit roundoff 2^-11, with an absolute floor of 2^-25 (half the
spacing of fp16's subnormals) for the smallest values.
"""
import math

import numpy as np
import pytest

import oracle.vmla_oracle as O
from latent_kv_attention_down_b200 import api, synth
from tests.harness import Rollout, sampled_rows, to_dev

pytestmark = pytest.mark.gpu

U_BF16 = 2.0 ** -8
U_F16 = 2.0 ** -11       # the reconstruct-once workspace holds fp16
F16_TINY = 2.0 ** -25    # half the spacing of fp16's subnormals: the absolute floor of its rounding


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


# ------------------------------------------------------------------ reading the GPU's buffers

def bf16_view(t, shape, dtype=None):
    import torch
    dt = dtype or torch.bfloat16
    return t.view(dt)[: int(np.prod(shape))].view(*shape).float().cpu().numpy().astype(np.float64)


def ring(ro, layer=0):
    """The stored latent cache and positional keys of a layer: [B][W*T_f][d_c], [B][W*T_f][d_rope]."""
    d = ro.dims
    R = d.window_tokens
    n_c, n_r = d.batch * R * d.d_latent, d.batch * R * d.d_rope
    ckv = bf16_view(ro.m.ckv[layer * n_c * 2:(layer + 1) * n_c * 2], (d.batch, R, d.d_latent))
    kr = bf16_view(ro.m.kr[layer * n_r * 2:(layer + 1) * n_r * 2], (d.batch, R, d.d_rope))
    return ckv, kr


def workspace(ro, region, shape, fp16=False):
    import torch
    off = api.workspace_offsets(ro.cfg)[region]
    return bf16_view(ro.m.workspace[off:], shape, torch.float16 if fp16 else None)


def slot_positions(ro, frames_appended):
    """(t, h, w) of every ring row [0, n_keys) as the kernels see it: ring slot s holds window frame
    of slot s, whose t vmla_window reports."""
    d = ro.dims
    frames, slots, ts = ro.m.window(frames_appended)
    T = d.tokens_per_frame
    tok = np.arange(T)
    pos = np.zeros((len(slots) * T, 3), np.int64)
    for s, t in zip(slots, ts):
        pos[s * T:(s + 1) * T] = np.stack([np.full(T, t), tok // d.grid_w, tok % d.grid_w], axis=1)
    return pos, frames, ts


def query_positions(d, first, t_of_first):
    tok = np.arange(d.tokens_per_frame)
    rows = [np.stack([np.full_like(tok, t_of_first + k), tok // d.grid_w, tok % d.grid_w], axis=1)
            for k in range(d.chunk_frames)]
    return np.concatenate(rows).astype(np.int64)


def freqs_of(d):
    return O.rope_frequencies(d.rope_pairs, d.rope_theta, d.rope_base_dims)


def assert_rounded_once(got, ref, terms, what, u=U_BF16, floor=1e-30):
    """got = round(ref computed in fp32): |got - ref| <= u |ref| + 2^-20 * sum |terms| (+ floor, the
    absolute rounding of fp16's subnormal range)."""
    bound = u * np.abs(ref) + 2.0 ** -20 * terms + floor
    excess = np.abs(got - ref) - bound
    assert np.all(excess <= 0), f"{what}: worst excess {excess.max():.3e} (|err| {np.abs(got - ref).max():.3e})"


def attention_core_check(q, k, v, got, what, w_out=None, u=U_BF16, p_floor=0.0):
    """Textbook softmax attention (fp64) of queries q [M, d] over keys k [N, d] with values v [N, e]
    (then times w_out^T [e', e] when given), against the kernel's output got [M, e'] at the
    6-sigma P-rounding bound (relative rounding u of P, or at least p_floor absolute where P is
    subnormal in fp16).  Returns (max |err| / sigma, max |err| / RMS)."""
    scale = 1.0 / math.sqrt(128.0)
    vv = v if w_out is None else v @ w_out.T          # the per-key values reaching the output
    ref = np.zeros((q.shape[0], vv.shape[1]))
    var = np.zeros_like(ref)
    for b0 in range(0, q.shape[0], 512):
        s = (q[b0:b0 + 512] @ k.T) * scale
        s -= s.max(axis=1, keepdims=True)
        p = np.exp(s)
        l = p.sum(axis=1, keepdims=True)
        p /= l
        ref[b0:b0 + 512] = p @ vv
        # the rounding of each unnormalised p_j (at most 1 here; the kernel's, taken against its
        # running max, are no smaller, so p_floor / l overstates their subnormal share): u p_j, or
        # the absolute floor where p_j is subnormal
        dp = np.maximum(u * p, p_floor / l)
        var[b0:b0 + 512] = (dp * dp) @ (vv * vv)
    sigma = np.sqrt(var / 3.0)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    err = np.abs(got - ref)
    bound = 6.0 * sigma + 1e-4 * rms
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert np.all(err <= bound), (f"{what}: element {worst} err {err[worst]:.3e} > 6 sigma {6 * sigma[worst]:.3e} "
                                  f"+ {1e-4 * rms:.3e}")
    return float(np.max(err / (sigma + 1e-30))), float(err.max() / rms)


# ------------------------------------------------------------------ the stages

def _rollout(d, chunks, design):
    ro = Rollout(d, design=api.DESIGN_RECON_ONCE)  # workspace with room for every design's intermediates
    for c in range(chunks):
        ro.append_chunk(0, c)
    out, q = ro.attend(0, chunks - 1, design=design)
    return ro, out, q


def _split(d_rope, d_latent=192):
    d_nope, pairs = {16: (112, (4, 2, 2)), 64: (64, (12, 10, 10)), 96: (32, (16, 16, 16))}[d_rope]
    return synth.WAN_SMALL.replace(name=f"wan_small_r{d_rope}_c{d_latent}", d_nope=d_nope, d_rope=d_rope,
                                   rope_pairs=pairs, d_latent=d_latent)


# the Wan-1.3B layer and its 10x20 grid (96/32 split): first chunk, full window, wrapped ring; the
# 112/16, 64/64 and 32/96 splits on the full small window
CASES = [(synth.WAN_SMALL, 1), (synth.WAN_SMALL, 7), (synth.WAN_SMALL, 10), (synth.WAN, 7),
         (_split(16), 7), (_split(64), 7), (_split(96), 7)]


def _grid(h, w):
    return synth.WAN_SMALL.replace(name=f"wan_grid{h}x{w}", grid_h=h, grid_w=w)


# Windows whose last 192-key tile of the per-head kernel ends at each softmax group's edge (each
# group takes 96 of a tile's keys): 96 keys (the second group's half empty), 192 (one full tile),
# 195 (3 keys past it), 291 (the second group's half holding 3 keys), 672 (three tiles and an
# empty half); 96, 195 and 291 queries make one to three ragged query tiles.
TILE_EDGE_CASES = [(_grid(4, 8), 1), (_grid(4, 8), 2), (_grid(4, 8), 7), (_grid(5, 13), 1), (_grid(1, 97), 1)]


@pytest.mark.parametrize("dims,chunks", CASES, ids=lambda v: getattr(v, "name", v))
def test_stages_of_the_absorbed_design(dims, chunks):
    """Window RoPE, q-absorb and the absorbed attention core (with the fused W_uv) each against the
    fp64 definition fed the GPU's inputs of that stage; every query row of the small grid, 512
    seeded rows of every head of the Wan layer."""
    d = dims
    ro, out, q = _rollout(d, chunks, api.DESIGN_ABSORBED)
    F = chunks * d.chunk_frames
    first = F - d.chunk_frames
    w = ro.w[0]
    ckv, kr = ring(ro)
    pos, frames, ts = slot_positions(ro, F)
    n_keys = len(frames) * d.tokens_per_frame
    fr = freqs_of(d)

    # window RoPE: stored k_R rotated at the window-relative positions
    kr_rot = workspace(ro, api.WS_KR_ROT, (d.batch, d.window_tokens, d.d_rope))[0, :n_keys]
    ang = O.rope_angles(pos[:n_keys, 0], pos[:n_keys, 1], pos[:n_keys, 2], fr)
    ref = O.rope_rotate(kr[0, :n_keys], ang)
    pair = np.repeat(np.sqrt(kr[0, :n_keys, 0::2] ** 2 + kr[0, :n_keys, 1::2] ** 2), 2, axis=1)
    assert_rounded_once(kr_rot, ref, 16 * pair, "window RoPE")

    # q-absorb: q~_h = [W_uk,h^T q_nope | RoPE(q_rope)] at the chunk's positions
    nq, dqk = d.n_queries, d.d_latent + d.d_rope
    qt = workspace(ro, api.WS_QT, (d.batch, d.n_heads, nq, dqk))[0]
    t_first = ts[frames.index(first)]
    qpos = query_positions(d, first, t_first)
    rows = np.arange(nq) if nq <= 1024 else sampled_rows(nq, 512, seed=chunks)
    qa = q[0][rows]
    qrot = O.rotate_queries(qa, qpos[rows], d.d_nope, fr)
    for h in range(d.n_heads):
        lat = qa[:, h, :d.d_nope] @ w.w_uk[h]
        terms = np.abs(qa[:, h, :d.d_nope]) @ np.abs(w.w_uk[h])
        assert_rounded_once(qt[h][rows, :d.d_latent], lat, terms, f"q-absorb latent part, head {h}")
        rp = qrot[:, h, d.d_nope:]
        assert_rounded_once(qt[h][rows, d.d_latent:], rp, 16 * np.abs(qa[:, h, d.d_nope:]).max(), f"q rope, head {h}")

    # attention core over the GPU's q~, [c | k_R rotated] and c, then W_uv,h
    key = np.concatenate([ckv[0, :n_keys], kr_rot], axis=1)
    worst = []
    for h in range(d.n_heads):
        got = out[0][rows, h * d.d_head:(h + 1) * d.d_head]
        worst.append(attention_core_check(qt[h][rows], key, ckv[0, :n_keys], got, f"absorbed core, head {h}",
                                          w_out=w.w_uv[h]))
    print(f"absorbed core {d.name} {chunks} chunks: max err/sigma {max(x[0] for x in worst):.2f}, "
          f"max err/rms {max(x[1] for x in worst):.2e}")


@pytest.mark.parametrize("dims,chunks", CASES + TILE_EDGE_CASES, ids=lambda v: getattr(v, "name", v))
def test_stages_of_the_reconstruct_once_design(dims, chunks):
    """Per-head queries, the reconstruction of the window's per-head K/V and the d_head = 128
    attention core, each against the fp64 definition fed the GPU's inputs of that stage."""
    d = dims
    ro, out, q = _rollout(d, chunks, api.DESIGN_RECON_ONCE)
    F = chunks * d.chunk_frames
    first = F - d.chunk_frames
    w = ro.w[0]
    ckv, kr = ring(ro)
    pos, frames, ts = slot_positions(ro, F)
    n_keys = len(frames) * d.tokens_per_frame
    fr = freqs_of(d)
    # the window's positional keys, rotated for this call by the reconstruction and kept in fp16 in
    # every head's key (head 0's copy here; the others must equal it)
    recon = workspace(ro, api.WS_RECON, (d.batch, d.window_tokens, 2, d.n_heads, d.d_head), fp16=True)[0, :n_keys]
    kr_rot = recon[:, 0, 0, d.d_nope:]
    ang = O.rope_angles(pos[:n_keys, 0], pos[:n_keys, 1], pos[:n_keys, 2], fr)
    pair = np.repeat(np.sqrt(kr[0, :n_keys, 0::2] ** 2 + kr[0, :n_keys, 1::2] ** 2), 2, axis=1)
    assert_rounded_once(kr_rot, O.rope_rotate(kr[0, :n_keys], ang), 16 * pair, "window RoPE (fp16)", u=U_F16,
                        floor=F16_TINY)

    # per-head queries in fp16: content part converted (exact but for fp16 subnormals), positional
    # part rotated and rounded once
    nq = d.n_queries
    qd = workspace(ro, api.WS_QD, (d.batch, d.n_heads, nq, d.d_head), fp16=True)[0]
    t_first = ts[frames.index(first)]
    qpos = query_positions(d, first, t_first)
    rows = np.arange(nq) if nq <= 1024 else sampled_rows(nq, 512, seed=chunks)
    qa = q[0][rows]
    qrot = O.rotate_queries(qa, qpos[rows], d.d_nope, fr)
    for h in range(d.n_heads):
        assert_rounded_once(qd[h][rows, :d.d_nope], qa[:, h, :d.d_nope], 0.0, f"q content, head {h}", u=0.0,
                            floor=F16_TINY)
        assert_rounded_once(qd[h][rows, d.d_nope:], qrot[:, h, d.d_nope:], 16 * np.abs(qa[:, h, d.d_nope:]).max(),
                            f"q rope, head {h}", u=U_F16, floor=F16_TINY)

    # reconstruction in fp16: K_h = [W_uk,h c | k_R rotated], V_h = W_uv,h c from the stored cache
    c = ckv[0, :n_keys]
    keys = np.arange(n_keys) if n_keys <= 8192 else np.sort(np.random.default_rng(1).choice(n_keys, 8192, False))
    for h in range(d.n_heads):
        kn = c[keys] @ w.w_uk[h].T
        assert_rounded_once(recon[keys, 0, h, :d.d_nope], kn, np.abs(c[keys]) @ np.abs(w.w_uk[h]).T,
                            f"K content, head {h}", u=U_F16, floor=F16_TINY)
        assert_rounded_once(recon[:, 0, h, d.d_nope:], kr_rot, 0.0, f"K positional copy, head {h}", u=0.0,
                            floor=F16_TINY)
        vv = c[keys] @ w.w_uv[h].T
        assert_rounded_once(recon[keys, 1, h], vv, np.abs(c[keys]) @ np.abs(w.w_uv[h]).T, f"V, head {h}",
                            u=U_F16, floor=F16_TINY)

    # attention core over the GPU's per-head q, K_h and V_h (P rounded to fp16)
    worst = []
    for h in range(d.n_heads):
        got = out[0][rows, h * d.d_head:(h + 1) * d.d_head]
        worst.append(attention_core_check(qd[h][rows], recon[:, 0, h], recon[:, 1, h], got,
                                          f"per-head core, head {h}", u=U_F16, p_floor=F16_TINY))
    print(f"per-head core {d.name} {chunks} chunks: max err/sigma {max(x[0] for x in worst):.2f}, "
          f"max err/rms {max(x[1] for x in worst):.2e}")


@pytest.mark.parametrize("dims,chunks", [(synth.WAN_SMALL, 1), (synth.WAN_SMALL, 7)] + TILE_EDGE_CASES[1:4:2],
                         ids=lambda v: getattr(v, "name", v))
def test_stages_of_the_dense_comparison(dims, chunks):
    """The dense per-head cache (3072 scalars per token): its stored keys and values against the
    fp64 reconstruction from x's bf16 latents, and the attention core over the stored entries."""
    d = dims
    ro = Rollout(d, dense=True)
    for c in range(chunks):
        ro.append_chunk(0, c, dense=True)
    out, q = ro.attend(0, chunks - 1, dense=True)
    F = chunks * d.chunk_frames
    first = F - d.chunk_frames
    w = ro.w[0]
    R, n_keys = d.window_tokens, min(F, d.window_frames) * d.tokens_per_frame
    dense = bf16_view(ro.m.dense_kv, (d.batch, R, 2, d.n_heads, d.d_head))[0, :n_keys]
    nq = d.n_queries
    qd = workspace(ro, api.WS_QD, (d.batch, d.n_heads, nq, d.d_head))[0]
    fr = freqs_of(d)
    # queries and keys of the dense layout are rotated at absolute frame positions
    qpos = query_positions(d, first, first)
    qrot = O.rotate_queries(q[0], qpos, d.d_nope, fr)
    # stored entries: c = bf16(W_dkv x), then K_h = bf16([W_uk,h c | RoPE(bf16(W_kr x))]), V_h = bf16(W_uv,h c);
    # against the fp64 definition from x the two roundings give |err| <= u |ref| + u (|W| |c|) (+ fp32)
    T = d.tokens_per_frame
    for f in range(max(0, F - d.window_frames), F):
        rows_f = slice((f % d.window_frames) * T, (f % d.window_frames + 1) * T)
        c64, r64 = O.down_project(ro.frame_x[0][0][f], w.w_down, d.d_latent)
        ang = O.rope_angles(np.full(T, f), np.arange(T) // d.grid_w, np.arange(T) % d.grid_w, fr)
        kr_ref = O.rope_rotate(r64, ang)
        pair = np.repeat(np.sqrt(r64[:, 0::2] ** 2 + r64[:, 1::2] ** 2), 2, axis=1)
        for h in range(d.n_heads):
            kn, vv = c64 @ w.w_uk[h].T, c64 @ w.w_uv[h].T
            inner = U_BF16 / 2.0 ** -20  # the latent's own rounding, carried through the sum
            assert_rounded_once(dense[rows_f, 0, h, :d.d_nope], kn, inner * np.abs(c64) @ np.abs(w.w_uk[h]).T,
                                f"dense K content, frame {f} head {h}")
            assert_rounded_once(dense[rows_f, 1, h], vv, inner * np.abs(c64) @ np.abs(w.w_uv[h]).T,
                                f"dense V, frame {f} head {h}")
            assert_rounded_once(dense[rows_f, 0, h, d.d_nope:], kr_ref, inner * pair, f"dense K rope, frame {f}")
    for h in range(d.n_heads):
        assert np.array_equal(qd[h][:, :d.d_nope], q[0][:, h, :d.d_nope])
        assert_rounded_once(qd[h][:, d.d_nope:], qrot[:, h, d.d_nope:], 16 * np.abs(q[0][:, h, d.d_nope:]).max(),
                            f"dense q rope, head {h}")
    worst = []
    for h in range(d.n_heads):
        got = out[0][:, h * d.d_head:(h + 1) * d.d_head]
        worst.append(attention_core_check(qd[h], dense[:, 0, h], dense[:, 1, h], got, f"dense core, head {h}"))
    print(f"dense core {d.name} {chunks} chunks: max err/sigma {max(x[0] for x in worst):.2f}")
