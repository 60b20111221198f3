"""fp64 CPU oracle for VideoMLA latent-KV chunk attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this module:
only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may call it.  It shares no code with the CUDA library.

It is the plain, non-absorbed definition of the method, written out step by
step in float64 with numpy (a matrix product is the only library primitive it
leans on).  Sources, cited by page and section:

* [paperlayer] VideoMLA summary on paperlayer.ai -- §3 Method, §4, App. C.1,
  App. D.1-D.5, App. E;
* [gist.it] VideoMLA technical summary on gist.science (Italian),
  "Metodologia" points 1-4;
* [rp.zh] VideoMLA summary on researchpapers.dev (Chinese), key results.

Readings taken where the pages are silent (each one is listed with its
reason in the design notes of the repository):

* RoPE frequencies  w_{a,i} = theta^(-2 i / B_a), i = 0..n_a-1, with
  B_a = 2 n_a unless a larger per-axis band count is given (then the
  highest-frequency n_a bands of that group are used); pairs are adjacent
  (2i, 2i+1) dims, axis order t | h | w; token index = h * grid_w + w.
* softmax scale 1/sqrt(d_nope + d_rope); no norms; no mask (the queries are
  the newest chunk, which may see the whole window, itself included).
* the window holds the last ``window_frames`` frames, current chunk included;
  with the positional key stored before rotation, keys and queries get the
  window-relative frame index t = f - first_frame_of_window ("at read"), or
  the absolute frame index ("at append").
* k_R is projected from x (its own rows of W_down), not from c_KV.

Parity status: every function below is pinned by ``tests/test_oracle.py``
(closed forms, the numbers the pages print, invariants, brute force, and a
library attention routine).  The end-to-end model numbers of the pages
(1.23x throughput, 23.96 FPS, 8.0x batch) need the trained model and are
parity unpinned; this oracle does not compute them.
"""
from __future__ import annotations

import math
from collections.abc import Sequence

import numpy as np

# --------------------------------------------------------------------------
# Cache accounting  [gist.it pt. 4; paperlayer §3 "Cache efficiency", App. D.2,
# App. C.1; rp.zh key results]
# --------------------------------------------------------------------------


def latent_scalars_per_token(d_latent: int, d_rope: int) -> int:
    """Cached scalars per token per layer in the latent layout: d_c + d_rope."""
    return d_latent + d_rope


def dense_scalars_per_token(n_heads: int, d_head: int) -> int:
    """Cached scalars per token per layer in the per-head layout: 2 n_h d_h."""
    return 2 * n_heads * d_head


def cache_scalars(frames: int, tokens_per_frame: int, layers: int, scalars_per_token: int) -> int:
    return frames * tokens_per_frame * layers * scalars_per_token


# --------------------------------------------------------------------------
# Sliding window and ring slots  [paperlayer App. D.4 FIFO eviction; App. D.5
# window-relative coordinates; App. D.1 21 latent frames x 1560 tokens]
# --------------------------------------------------------------------------


def window_frame_range(frames_appended: int, window_frames: int) -> tuple[int, int]:
    """Frames [start, end) in the window after ``frames_appended`` frames were
    written: the newest ``window_frames`` of them (FIFO eviction)."""
    return max(0, frames_appended - window_frames), frames_appended


def window_frames_list(frames_appended: int, window_frames: int, sink_frames: int = 0) -> list[int]:
    """Frames in the active context after ``frames_appended`` frames, in cache
    order: the ``sink_frames`` first frames of the rollout stay for good, the
    other ``window_frames - sink_frames`` slots hold the newest frames, the
    oldest evicted first [paperlayer App. D.4: one sink latent frame and the
    six most recent latent frames, FIFO eviction outside the sink]."""
    F, S, W = frames_appended, sink_frames, window_frames
    sink = list(range(min(S, F)))
    local_start = max(S, F - (W - S))
    return sink + list(range(local_start, F))


def window_frame_t(frames_appended: int, window_frames: int, sink_frames: int = 0) -> dict:
    """Window-relative temporal coordinate of every frame of the active context
    [paperlayer App. D.5: cached positional keys get local temporal coordinates
    in the sink-plus-window context]: the sink frames keep 0..S-1, the local
    frames follow them in order, S, S+1, ... -- so t never exceeds
    window_frames - 1 however long the rollout."""
    frames = window_frames_list(frames_appended, window_frames, sink_frames)
    return {f: t for t, f in enumerate(frames)}


def ring_slot(frame: int, window_frames: int, sink_frames: int = 0) -> int:
    """Ring slot of a frame in a cache of ``window_frames`` frames: a sink frame
    keeps its own slot, any other frame takes the slot of the local frame it
    evicts (the oldest one)."""
    if frame < sink_frames:
        return frame
    return sink_frames + (frame - sink_frames) % (window_frames - sink_frames)


def token_grid_position(token: np.ndarray | int, grid_w: int):
    """(h, w) of a token index inside its latent frame (row-major grid)."""
    return np.asarray(token) // grid_w, np.asarray(token) % grid_w


# --------------------------------------------------------------------------
# 3D-RoPE  [paperlayer App. C.1: separate t/h/w subspaces, concatenated, max
# length 1024 per axis; App. D.3: 16 complex pairs as (6, 5, 5), highest-
# frequency bands of each axis group]
# --------------------------------------------------------------------------

ROPE_MAX_POSITION = 1024


def rope_frequencies(pairs: Sequence[int], theta: float = 10000.0,
                     base_dims: Sequence[int] | None = None) -> list[np.ndarray]:
    """Angular frequency of each complex pair, per axis (t, h, w).

    Axis a has n_a pairs; pair i turns at theta^(-2 i / B_a), where B_a is the
    number of rotary dims of that axis' band group (2 n_a by default).  i = 0
    is the highest frequency, so the first n_a bands are the highest ones."""
    out = []
    for a, n in enumerate(pairs):
        b = base_dims[a] if base_dims is not None and base_dims[a] else 2 * n
        i = np.arange(n, dtype=np.float64)
        out.append(np.power(float(theta), -2.0 * i / float(b)))
    return out


def rope_angles(t, h, w, freqs: list[np.ndarray]) -> np.ndarray:
    """Rotation angle of every pair for positions (t, h, w): [..., n_pairs],
    pairs ordered t-axis first, then h, then w."""
    t, h, w = (np.asarray(v, dtype=np.float64) for v in (t, h, w))
    return np.concatenate([np.multiply.outer(t, freqs[0]),
                           np.multiply.outer(h, freqs[1]),
                           np.multiply.outer(w, freqs[2])], axis=-1)


def rope_rotate(v: np.ndarray, angles: np.ndarray) -> np.ndarray:
    """Rotate each adjacent pair (v[2i], v[2i+1]) of the last axis by angles[..., i]."""
    v = np.asarray(v, dtype=np.float64)
    x0, x1 = v[..., 0::2], v[..., 1::2]
    c, s = np.cos(angles), np.sin(angles)
    y0 = x0 * c - x1 * s
    y1 = x0 * s + x1 * c
    return np.stack([y0, y1], axis=-1).reshape(y0.shape[:-1] + (2 * y0.shape[-1],))


# --------------------------------------------------------------------------
# Latent cache content  [gist.it pt. 1 (c_KV = W_down x), pt. 3 (one head-
# shared positional key k_R); paperlayer §3 "Shared low-rank KV cache"]
# --------------------------------------------------------------------------


def down_project(x: np.ndarray, w_down: np.ndarray, d_latent: int):
    """c_KV = W_dkv x and the unrotated positional key k_R = W_kr x, where
    W_down stacks W_dkv (first d_latent rows) over W_kr."""
    y = np.asarray(x, dtype=np.float64) @ np.asarray(w_down, dtype=np.float64).T
    return y[..., :d_latent], y[..., d_latent:]


def key_positions(frames: Sequence[int], t_origin: int, grid_h: int, grid_w: int) -> np.ndarray:
    """(t, h, w) of every token of ``frames`` (in order), t = frame - t_origin."""
    tok = np.arange(grid_h * grid_w)
    hh, ww = token_grid_position(tok, grid_w)
    rows = []
    for f in frames:
        rows.append(np.stack([np.full_like(tok, f - t_origin), hh, ww], axis=1))
    return np.concatenate(rows, axis=0).astype(np.int64)


# --------------------------------------------------------------------------
# Attention: the non-absorbed definition  [gist.it pt. 2 and 3; paperlayer §3
# "On-demand reconstruction", "Decoupled positional encoding", App. D.3-D.5]
# --------------------------------------------------------------------------


def reconstruct_heads(c: np.ndarray, k_rope: np.ndarray, w_uk: np.ndarray, w_uv: np.ndarray):
    """Per-head keys and values from the cached latent: k_h = [W_uk,h c | k_rope]
    (positional part shared by all heads) and v_h = W_uv,h c.
    Returns k [N, n_h, d_nope + d_rope], v [N, n_h, d_v]."""
    c = np.asarray(c, dtype=np.float64)
    n_h = w_uk.shape[0]
    k_nope = np.einsum("nc,hdc->nhd", c, np.asarray(w_uk, dtype=np.float64))
    k = np.concatenate([k_nope, np.broadcast_to(k_rope[:, None, :], (c.shape[0], n_h, k_rope.shape[1]))], axis=2)
    v = np.einsum("nc,hdc->nhd", c, np.asarray(w_uv, dtype=np.float64))
    return k, v


def softmax_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float) -> np.ndarray:
    """Textbook single-head attention: softmax(q k^T * scale) v, with the max
    subtracted before exponentiating.  q [M, d], k [N, d], v [N, e]."""
    s = (np.asarray(q, np.float64) @ np.asarray(k, np.float64).T) * scale
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=1, keepdims=True)
    return p @ np.asarray(v, np.float64)


def rotate_queries(q: np.ndarray, query_pos: np.ndarray, d_nope: int, freqs) -> np.ndarray:
    """q [N_q, n_h, d_nope + d_rope] -> same with the positional part rotated by
    each query's (t, h, w)."""
    q = np.asarray(q, dtype=np.float64)
    ang = rope_angles(query_pos[:, 0], query_pos[:, 1], query_pos[:, 2], freqs)  # [N_q, P]
    out = q.copy()
    out[..., d_nope:] = rope_rotate(q[..., d_nope:], ang[:, None, :])
    return out


def chunk_attention(c, r, key_pos, q, query_pos, w_uk, w_uv, *, d_nope, rope_pairs,
                    rope_theta=10000.0, rope_base_dims=None, query_rows=None, heads=None,
                    block=1024) -> np.ndarray:
    """Latent chunk attention, non-absorbed form.

    c [N_k, d_c] cached latents; r [N_k, d_rope] cached positional keys, NOT
    rotated; key_pos [N_k, 3] their (t, h, w); q [N_q, n_h, d_nope + d_rope]
    per-head queries with query_pos [N_q, 3]; w_uk [n_h, d_nope, d_c];
    w_uv [n_h, d_v, d_c].  Every key attends (no mask).

    Returns out [len(query_rows), n_h, d_v] (all rows by default), where
    out[i, h] = sum_j softmax_j(q_ih . k_jh / sqrt(d_nope + d_rope)) v_jh."""
    freqs = rope_frequencies(rope_pairs, rope_theta, rope_base_dims)
    key_pos = np.asarray(key_pos)
    k_rope = rope_rotate(r, rope_angles(key_pos[:, 0], key_pos[:, 1], key_pos[:, 2], freqs))
    rows = np.arange(q.shape[0]) if query_rows is None else np.asarray(query_rows)
    qr = rotate_queries(np.asarray(q)[rows], np.asarray(query_pos)[rows], d_nope, freqs)
    n_h = w_uk.shape[0]
    heads = range(n_h) if heads is None else heads
    scale = 1.0 / math.sqrt(qr.shape[2])
    out = np.zeros((len(rows), n_h, w_uv.shape[1]), dtype=np.float64)
    c64 = np.asarray(c, dtype=np.float64)
    for h in heads:
        k_h = np.concatenate([c64 @ np.asarray(w_uk[h], np.float64).T, k_rope], axis=1)
        v_h = c64 @ np.asarray(w_uv[h], np.float64).T
        for b0 in range(0, len(rows), block):
            out[b0:b0 + block, h] = softmax_attention(qr[b0:b0 + block, h], k_h, v_h, scale)
    return out


def chunk_attention_absorbed(c, r, key_pos, q, query_pos, w_uk, w_uv, *, d_nope, rope_pairs,
                             rope_theta=10000.0, rope_base_dims=None) -> np.ndarray:
    """The inference-time absorbed form [paperlayer App. E]: the content score
    uses the query pushed through W_uk (never the per-head keys), the value
    path accumulates softmax-weighted latents and applies W_uv afterwards.
    Used only to check the definition above, which it must equal."""
    freqs = rope_frequencies(rope_pairs, rope_theta, rope_base_dims)
    key_pos = np.asarray(key_pos)
    k_rope = rope_rotate(r, rope_angles(key_pos[:, 0], key_pos[:, 1], key_pos[:, 2], freqs))
    qr = rotate_queries(q, np.asarray(query_pos), d_nope, freqs)
    c64 = np.asarray(c, dtype=np.float64)
    key = np.concatenate([c64, k_rope], axis=1)  # shared by every head
    scale = 1.0 / math.sqrt(qr.shape[2])
    n_h = w_uk.shape[0]
    out = np.zeros((q.shape[0], n_h, w_uv.shape[1]))
    for h in range(n_h):
        q_lat = qr[:, h, :d_nope] @ np.asarray(w_uk[h], np.float64)  # W_uk,h^T q_nope
        q_tilde = np.concatenate([q_lat, qr[:, h, d_nope:]], axis=1)
        o_lat = softmax_attention(q_tilde, key, c64, scale)  # sum_j p_j c_j
        out[:, h] = o_lat @ np.asarray(w_uv[h], np.float64).T
    return out


def output_projection(o_heads: np.ndarray, w_o: np.ndarray) -> np.ndarray:
    """The layer's output mixer after attention: out = W_O [o_1 | ... | o_n_h] with
    o_heads [N, n_h, d_v] and W_O [d_out, n_h * d_v]."""
    o = np.asarray(o_heads, dtype=np.float64)
    return o.reshape(o.shape[0], -1) @ np.asarray(w_o, dtype=np.float64).T


def fold_output_weights(w_o: np.ndarray, w_uv: np.ndarray) -> np.ndarray:
    """B_h = W_O,h W_uv,h for every head, side by side: [d_out, n_h * d_c]
    [paperlayer App. E: the value path's W_uv,h is absorbed after accumulation,
    here all the way into the output mixer]."""
    n_h, d_v, d_c = w_uv.shape
    w_o = np.asarray(w_o, dtype=np.float64)
    return np.concatenate([w_o[:, h * d_v:(h + 1) * d_v] @ np.asarray(w_uv[h], np.float64) for h in range(n_h)],
                          axis=1)


def chunk_attention_folded(c, r, key_pos, q, query_pos, w_uk, w_fold, *, d_nope, rope_pairs,
                           rope_theta=10000.0, rope_base_dims=None) -> np.ndarray:
    """The absorbed form end to end: out = sum_h B_h o~_h with o~_h = sum_j p_hj c_j
    the softmax-weighted latents of head h and w_fold = [B_1 | ... | B_n_h].  Used
    only to check it against output_projection(chunk_attention(...), W_O)."""
    freqs = rope_frequencies(rope_pairs, rope_theta, rope_base_dims)
    key_pos = np.asarray(key_pos)
    k_rope = rope_rotate(r, rope_angles(key_pos[:, 0], key_pos[:, 1], key_pos[:, 2], freqs))
    qr = rotate_queries(q, np.asarray(query_pos), d_nope, freqs)
    c64 = np.asarray(c, dtype=np.float64)
    key = np.concatenate([c64, k_rope], axis=1)
    scale = 1.0 / math.sqrt(qr.shape[2])
    n_h, d_c = w_uk.shape[0], c64.shape[1]
    o_lat = np.zeros((q.shape[0], n_h * d_c))
    for h in range(n_h):
        q_tilde = np.concatenate([qr[:, h, :d_nope] @ np.asarray(w_uk[h], np.float64), qr[:, h, d_nope:]], axis=1)
        o_lat[:, h * d_c:(h + 1) * d_c] = softmax_attention(q_tilde, key, c64, scale)
    return o_lat @ np.asarray(w_fold, dtype=np.float64).T


def query_from_latent(c_q: np.ndarray, w_uq: np.ndarray, w_qr: np.ndarray) -> np.ndarray:
    """Per-head queries from the query latent c_Q [N, d_q] [paperlayer §4: d_q = 768]:
    q_h = [W_uq,h c_Q | W_qr,h c_Q] with w_uq [n_h, d_nope, d_q], w_qr [n_h, d_rope, d_q];
    returns [N, n_h, d_nope + d_rope] (positional part not yet rotated)."""
    c = np.asarray(c_q, dtype=np.float64)
    return np.concatenate([np.einsum("nj,hdj->nhd", c, np.asarray(w_uq, np.float64)),
                           np.einsum("nj,hdj->nhd", c, np.asarray(w_qr, np.float64))], axis=2)


def fold_query_weights(w_uq: np.ndarray, w_qr: np.ndarray, w_uk: np.ndarray) -> np.ndarray:
    """A_h = W_uk,h^T W_uq,h stacked over W_qr,h: [n_h, d_c + d_rope, d_q] [paperlayer App. E,
    content path absorbed into the query latent]."""
    a = np.einsum("hnc,hnj->hcj", np.asarray(w_uk, np.float64), np.asarray(w_uq, np.float64))
    return np.concatenate([a, np.asarray(w_qr, np.float64)], axis=1)


def chunk_attention_query_latent(c, r, key_pos, c_q, query_pos, w_qabs, w_uv, *, d_latent, d_head, rope_pairs,
                                 rope_theta=10000.0, rope_base_dims=None) -> np.ndarray:
    """The absorbed form fed from the query latent: q~_h = [A_h c_Q | RoPE(W_qr,h c_Q)]
    (w_qabs from fold_query_weights) against the shared key [c | RoPE(k_R)].  Used only to
    check it against chunk_attention(query_from_latent(...))."""
    freqs = rope_frequencies(rope_pairs, rope_theta, rope_base_dims)
    key_pos = np.asarray(key_pos)
    qpos = np.asarray(query_pos)
    k_rope = rope_rotate(r, rope_angles(key_pos[:, 0], key_pos[:, 1], key_pos[:, 2], freqs))
    c64 = np.asarray(c, dtype=np.float64)
    key = np.concatenate([c64, k_rope], axis=1)
    d_rope = key.shape[1] - d_latent
    scale = 1.0 / math.sqrt(d_head)  # the per-head score is a (d_nope + d_rope)-dim dot product
    n_h = w_qabs.shape[0]
    cq = np.asarray(c_q, dtype=np.float64)
    out = np.zeros((cq.shape[0], n_h, w_uv.shape[1]))
    for h in range(n_h):
        qt = cq @ np.asarray(w_qabs[h], np.float64).T
        qt[:, d_latent:] = rope_rotate(qt[:, d_latent:], rope_angles(qpos[:, 0], qpos[:, 1], qpos[:, 2], freqs))
        out[:, h] = softmax_attention(qt, key, c64, scale) @ np.asarray(w_uv[h], np.float64).T
    assert d_rope == 2 * sum(rope_pairs)
    return out


def dense_cache_entries(c, r, key_pos, w_uk, w_uv, *, rope_pairs, rope_theta=10000.0,
                        rope_base_dims=None):
    """The per-head dense layout of the same keys and values (2 n_h d_h scalars
    per token): rotated k_h = [W_uk,h c | RoPE(k_R)] and v_h = W_uv,h c."""
    freqs = rope_frequencies(rope_pairs, rope_theta, rope_base_dims)
    key_pos = np.asarray(key_pos)
    k_rope = rope_rotate(r, rope_angles(key_pos[:, 0], key_pos[:, 1], key_pos[:, 2], freqs))
    return reconstruct_heads(c, k_rope, w_uk, w_uv)


# --------------------------------------------------------------------------
# A rollout scenario: which frames are in the window, with which positions
# --------------------------------------------------------------------------


def window_latents(frame_x: dict, frames_appended: int, window_frames: int, w_down, d_latent,
                   grid_h: int, grid_w: int, rope_at: str = "read", sink_frames: int = 0):
    """Latents of the active context after ``frames_appended`` frames: the sink
    frames, then the local frames oldest first.

    frame_x maps a frame index to the x rows [tokens_per_frame, d_model] it
    was last appended with.  rope_at="read" gives every frame its
    window-relative t ([paperlayer App. D.5], ``window_frame_t``); "append"
    keeps the absolute frame index.  Returns (c, r, key_pos, t_origin), where
    a local frame f has t = f - t_origin (the chunk's queries use it)."""
    frames = window_frames_list(frames_appended, window_frames, sink_frames)
    x = np.concatenate([np.asarray(frame_x[f], dtype=np.float64) for f in frames], axis=0)
    c, r = down_project(x, w_down, d_latent)
    if rope_at == "read":
        t_of = window_frame_t(frames_appended, window_frames, sink_frames)
        t_origin = frames[-1] - t_of[frames[-1]]
    else:
        t_of = {f: f for f in frames}
        t_origin = 0
    tok = np.arange(grid_h * grid_w)
    hh, ww = token_grid_position(tok, grid_w)
    pos = np.concatenate([np.stack([np.full_like(tok, t_of[f]), hh, ww], axis=1) for f in frames], axis=0)
    return c, r, pos.astype(np.int64), t_origin


def chunk_query_positions(first_frame: int, n_frames: int, t_origin: int, grid_h: int, grid_w: int):
    return key_positions(range(first_frame, first_frame + n_frames), t_origin, grid_h, grid_w)
