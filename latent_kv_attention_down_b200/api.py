"""ctypes binding of libvmla.so (include/vmla.h): argument marshalling only.

Every computation runs in the library's CUDA kernels.  PyTorch is used for
device memory and streams: tensors are passed as raw device pointers with the
current CUDA stream.  If the library is not built, loading it raises.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libvmla.so")

c_int, c_float, c_size_t, c_int64, c_uint32, c_uint64, c_void_p, c_double = (
    ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_int64, ctypes.c_uint32, ctypes.c_uint64,
    ctypes.c_void_p, ctypes.c_double)

BF16, FP32 = 0, 1
DESIGN_AUTO, DESIGN_ABSORBED, DESIGN_RECONSTRUCT, DESIGN_RECON_ONCE = 0, 1, 2, 3
ROPE_AT_READ, ROPE_AT_APPEND = 0, 1
STAGES = {"append": 0, "rope": 1, "q_absorb": 2, "attention": 3, "attention_reconstruct": 4,
          "dense_append": 5, "dense_attention": 6, "reconstruct_once": 7, "folded_mixer": 8}


ABI_VERSION = 3  # VMLA_ABI_VERSION of include/vmla.h that this binding's structures follow


class Config(ctypes.Structure):
    """vmla_config of include/vmla.h, field for field."""
    _fields_ = [("d_model", c_int), ("n_heads", c_int), ("d_nope", c_int), ("d_rope", c_int),
                ("d_latent", c_int), ("d_value", c_int), ("rope_pairs", c_int * 3), ("rope_base_dims", c_int * 3),
                ("rope_theta", c_float), ("grid_h", c_int), ("grid_w", c_int), ("window_frames", c_int),
                ("chunk_frames", c_int), ("batch", c_int), ("layers", c_int), ("dtype", c_int),
                ("rope_mode", c_int), ("softmax_rescale_log2", c_float), ("sink_frames", c_int)]


class VmlaError(RuntimeError):
    """A vmla_status other than VMLA_OK, with its name (and the CUDA error behind VMLA_ERR_CUDA)."""
    def __init__(self, status: int, what: str):
        self.status = status
        msg = f"{what}: {lib().vmla_status_string(status).decode()}"
        if status == 4:  # VMLA_ERR_CUDA: say which CUDA error
            msg += f" ({lib().vmla_last_error_detail().decode()})"
        super().__init__(msg)


_SIGS = {
    "vmla_status_string": (ctypes.c_char_p, [c_int]),
    "vmla_last_error_detail": (ctypes.c_char_p, []),
    "vmla_abi_version": (c_int, []),
    "vmla_config_init": (c_int, [ctypes.POINTER(Config)]),
    "vmla_config_check": (c_int, [ctypes.POINTER(Config)]),
    "vmla_cache_bytes": (c_int, [ctypes.POINTER(Config), ctypes.POINTER(c_size_t), ctypes.POINTER(c_size_t),
                                 ctypes.POINTER(c_size_t)]),
    "vmla_workspace_bytes": (c_int, [ctypes.POINTER(Config), c_int, ctypes.POINTER(c_size_t)]),
    "vmla_rope_frequencies": (c_int, [ctypes.POINTER(Config), ctypes.POINTER(c_float), c_int]),
    "vmla_workspace_offsets": (c_int, [ctypes.POINTER(Config), ctypes.POINTER(c_size_t), c_int]),
    "vmla_create": (c_int, [ctypes.POINTER(Config), ctypes.POINTER(c_void_p)]),
    "vmla_destroy": (c_int, [c_void_p]),
    "vmla_bind": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_size_t]),
    "vmla_dense_bind": (c_int, [c_void_p, c_void_p]),
    "vmla_cache_append": (c_int, [c_void_p, c_int, c_void_p, c_void_p, c_int64, c_int, c_void_p]),
    "vmla_chunk_attention": (c_int, [c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_int, c_int,
                                     c_void_p]),
    "vmla_dense_cache_append": (c_int, [c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_int,
                                        c_void_p]),
    "vmla_dense_chunk_attention": (c_int, [c_void_p, c_int, c_void_p, c_void_p, c_int64, c_int, c_void_p]),
    "vmla_chunk_step_host": (c_int, [c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                     c_void_p, c_void_p, c_void_p, c_int64, c_int, c_int, c_void_p]),
    "vmla_window": (c_int, [c_void_p, c_int64, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32),
                            ctypes.POINTER(ctypes.c_int32), c_int, ctypes.POINTER(c_int)]),
    "vmla_state_get": (c_int, [c_void_p, c_int, ctypes.POINTER(c_int64)]),
    "vmla_state_set": (c_int, [c_void_p, c_int, c_int64]),
    "vmla_device_status": (c_int, [c_void_p, c_void_p, ctypes.POINTER(c_uint32)]),
    "vmla_profile_enable": (c_int, [c_void_p, c_int]),
    "vmla_set_append_tiling": (c_int, [c_void_p, c_int, c_int, c_int]),
    "vmla_fold_query_weights": (c_int, [ctypes.POINTER(Config), c_void_p, c_void_p, c_void_p, c_int, c_void_p,
                                        c_void_p]),
    "vmla_chunk_attention_qlatent": (c_int, [c_void_p, c_int, c_void_p, c_void_p, c_int, c_void_p, c_void_p,
                                             c_int64, c_int, c_void_p]),
    "vmla_fold_output_weights": (c_int, [ctypes.POINTER(Config), c_void_p, c_void_p, c_void_p, c_int, c_void_p]),
    "vmla_chunk_attention_folded": (c_int, [c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_int, c_void_p, c_int64,
                                            c_int, c_void_p]),
    "vmla_selftest_exp2": (c_int, [c_void_p, c_void_p, ctypes.c_int64, c_void_p]),
    "vmla_profile_read": (c_int, [c_void_p, c_int, ctypes.POINTER(c_double), ctypes.POINTER(c_int)]),
    "vmla_selftest_wait_timeout": (c_int, [c_uint64, c_void_p]),
    "vmla_chunk_attention_noalloc": (c_int, [ctypes.POINTER(Config), c_int, c_void_p, c_void_p, c_int64, c_void_p,
                                             c_void_p, c_void_p, c_void_p, c_int64, c_int, c_void_p]),
}

_LIB = None


def lib() -> ctypes.CDLL:
    """The loaded libvmla.so (loaded once).  Raises if it has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m latent_kv_attention_down_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        if handle.vmla_abi_version() != ABI_VERSION:
            raise RuntimeError(f"{LIB_PATH} has ABI version {handle.vmla_abi_version()}, this binding needs "
                               f"{ABI_VERSION}: rebuild it")
        _LIB = handle
    return _LIB


def check(status: int, what: str) -> None:
    """Raise VmlaError unless `status` is VMLA_OK."""
    if status != 0:
        raise VmlaError(status, what)


def config_from_dims(dims, layers: int = 1, rope_mode: int = ROPE_AT_READ) -> Config:
    """A vmla_config from a ``synth.Dims`` workload description."""
    c = Config()
    c.d_model, c.n_heads, c.d_nope, c.d_rope = dims.d_model, dims.n_heads, dims.d_nope, dims.d_rope
    c.d_latent, c.d_value = dims.d_latent, dims.d_head
    c.rope_pairs[:] = list(dims.rope_pairs)
    c.rope_base_dims[:] = list(dims.rope_base_dims)
    c.rope_theta = dims.rope_theta
    c.grid_h, c.grid_w = dims.grid_h, dims.grid_w
    c.window_frames, c.chunk_frames = dims.window_frames, dims.chunk_frames
    c.batch, c.layers = dims.batch, layers
    c.dtype = BF16 if dims.dtype == "bf16" else FP32
    c.rope_mode = rope_mode
    c.softmax_rescale_log2 = 8.0
    c.sink_frames = dims.sink_frames
    return c


def cache_bytes(cfg: Config):
    """vmla_cache_bytes: (latent cache, positional keys, dense per-head cache) bytes of a handle."""
    a, b, d = c_size_t(), c_size_t(), c_size_t()
    check(lib().vmla_cache_bytes(ctypes.byref(cfg), ctypes.byref(a), ctypes.byref(b), ctypes.byref(d)),
          "vmla_cache_bytes")
    return a.value, b.value, d.value


def workspace_bytes(cfg: Config, design: int = DESIGN_AUTO) -> int:
    """vmla_workspace_bytes: device workspace a handle needs for `design`."""
    n = c_size_t()
    check(lib().vmla_workspace_bytes(ctypes.byref(cfg), design, ctypes.byref(n)), "vmla_workspace_bytes")
    return n.value


WS_KR_ROT, WS_QT, WS_QD, WS_RECON = 0, 1, 2, 3


def workspace_offsets(cfg: Config):
    """vmla_workspace_offsets: byte offsets of the rotated window keys, absorbed queries, per-head
    queries and per-head K/V inside the workspace (indexed by WS_*)."""
    buf = (c_size_t * 4)()
    check(lib().vmla_workspace_offsets(ctypes.byref(cfg), buf, 4), "vmla_workspace_offsets")
    return list(buf)


def rope_frequencies(cfg: Config):
    """vmla_rope_frequencies: angular frequency of every rotary pair, t pairs first."""
    n = cfg.d_rope // 2
    buf = (c_float * max(n, 1))()
    check(lib().vmla_rope_frequencies(ctypes.byref(cfg), buf, max(n, 1)), "vmla_rope_frequencies")
    return list(buf)[:n]


def _ptr(t) -> int:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libvmla must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


class LatentKVAttention:
    """One vmla handle: the latent (and optionally dense) caches of ``cfg.layers``
    layers of ``cfg.batch`` samples, plus its workspace."""

    def __init__(self, cfg: Config):
        self.cfg = cfg
        h = c_void_p()
        check(lib().vmla_create(ctypes.byref(cfg), ctypes.byref(h)), "vmla_create")
        self._h = h
        self._keep = []

    def close(self):
        """vmla_destroy (idempotent)."""
        if getattr(self, "_h", None):
            lib().vmla_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -------------------------------------------------------------- memory
    def allocate(self, device="cuda", design: int = DESIGN_AUTO, dense: bool = False):
        """Allocate the caches and workspace with torch on ``device`` and bind them."""
        import torch
        ckv_b, kr_b, dense_b = cache_bytes(self.cfg)
        ws_b = workspace_bytes(self.cfg, design)
        self.ckv = torch.empty(ckv_b, dtype=torch.uint8, device=device)
        self.kr = torch.empty(kr_b, dtype=torch.uint8, device=device)
        self.workspace = torch.empty(max(ws_b, 256), dtype=torch.uint8, device=device)
        self.bind(self.ckv, self.kr, self.workspace)
        if dense:
            self.dense_kv = torch.empty(dense_b, dtype=torch.uint8, device=device)
            self.dense_bind(self.dense_kv)
        return self

    def bind(self, ckv, kr, workspace):
        """vmla_bind: attach caller-allocated caches and workspace (uint8 device tensors)."""
        check(lib().vmla_bind(self._h, _ptr(ckv), _ptr(kr), _ptr(workspace), workspace.numel() * workspace.element_size()),
              "vmla_bind")
        self._keep = [ckv, kr, workspace]

    def dense_bind(self, dense_kv):
        """vmla_dense_bind: attach the dense per-head cache."""
        check(lib().vmla_dense_bind(self._h, _ptr(dense_kv)), "vmla_dense_bind")
        self._keep.append(dense_kv)

    # -------------------------------------------------------------- compute
    def append(self, layer, x, w_down, first_frame, n_frames, stream=None):
        """vmla_cache_append: x [B][n_frames*T_f][d_model], w_down [d_c + d_rope][d_model]."""
        check(lib().vmla_cache_append(self._h, layer, _ptr(x), _ptr(w_down), first_frame, n_frames, _stream(stream)),
              "vmla_cache_append")

    def attention(self, layer, q, w_uk, w_uv, out, first_frame, n_frames, design=DESIGN_AUTO, stream=None):
        """vmla_chunk_attention: q [B][rows][n_h][d_head], w_uk [n_h][d_nope][d_c], w_uv [n_h][d_head][d_c], out fp32 [B][rows][n_h*d_head]."""
        check(lib().vmla_chunk_attention(self._h, layer, _ptr(q), _ptr(w_uk), _ptr(w_uv), _ptr(out), first_frame,
                                         n_frames, design, _stream(stream)), "vmla_chunk_attention")

    def dense_append(self, layer, x, w_down, w_uk, w_uv, first_frame, n_frames, stream=None):
        """vmla_dense_cache_append: per-head K/V of the chunk into the dense cache."""
        check(lib().vmla_dense_cache_append(self._h, layer, _ptr(x), _ptr(w_down), _ptr(w_uk), _ptr(w_uv),
                                            first_frame, n_frames, _stream(stream)), "vmla_dense_cache_append")

    def dense_attention(self, layer, q, out, first_frame, n_frames, stream=None):
        """vmla_dense_chunk_attention: d_head attention over the dense per-head cache."""
        check(lib().vmla_dense_chunk_attention(self._h, layer, _ptr(q), _ptr(out), first_frame, n_frames,
                                               _stream(stream)), "vmla_dense_chunk_attention")

    def step_host(self, layer, x_host, q_host, out_host, w_down, w_uk, w_uv, x_dev, q_dev, out_dev, first_frame,
                  n_frames, design=DESIGN_AUTO, stream=None):
        """vmla_chunk_step_host: append + attention from pinned host x, q into pinned host out, through
        the caller's device staging buffers; out_host is complete once `stream` reaches this call."""
        check(lib().vmla_chunk_step_host(self._h, layer, _ptr(x_host), _ptr(q_host), _ptr(out_host), _ptr(w_down),
                                         _ptr(w_uk), _ptr(w_uv), _ptr(x_dev), _ptr(q_dev), _ptr(out_dev),
                                         first_frame, n_frames, design, _stream(stream)), "vmla_chunk_step_host")

    # -------------------------------------------------------------- bookkeeping
    def window(self, frames_appended: int):
        """vmla_window: (frames, ring slots, window-relative t) of the window, sink frames first."""
        cap = self.cfg.window_frames
        f, s, t = (ctypes.c_int32 * cap)(), (ctypes.c_int32 * cap)(), (ctypes.c_int32 * cap)()
        n = c_int()
        check(lib().vmla_window(self._h, frames_appended, f, s, t, cap, ctypes.byref(n)), "vmla_window")
        return list(f)[:n.value], list(s)[:n.value], list(t)[:n.value]

    def state_get(self, layer: int) -> int:
        """vmla_state_get: frames appended so far to `layer` (resume point)."""
        v = c_int64()
        check(lib().vmla_state_get(self._h, layer, ctypes.byref(v)), "vmla_state_get")
        return v.value

    def state_set(self, layer: int, frames_appended: int):
        """vmla_state_set: resume `layer` at `frames_appended`."""
        check(lib().vmla_state_set(self._h, layer, frames_appended), "vmla_state_set")

    def device_status(self, stream=None):
        """(status, raw flag bits); synchronises the stream."""
        flags = c_uint32()
        st = lib().vmla_device_status(self._h, _stream(stream), ctypes.byref(flags))
        return st, flags.value

    def fold_query_weights(self, w_uq, w_qr, w_uk, w_qabs, stream=None):
        """w_qabs [n_h][d_c + d_rope][d_q] = [W_uk,h^T W_uq,h ; W_qr,h]."""
        check(lib().vmla_fold_query_weights(ctypes.byref(self.cfg), _ptr(w_uq), _ptr(w_qr), _ptr(w_uk),
                                            w_qabs.shape[2], _ptr(w_qabs), _stream(stream)), "vmla_fold_query_weights")

    def attention_qlatent(self, layer, c_q, w_qabs, w_uv, out, first_frame, n_frames, stream=None):
        """Absorbed chunk attention whose queries come from the query latent c_Q [B][rows][d_q]."""
        check(lib().vmla_chunk_attention_qlatent(self._h, layer, _ptr(c_q), _ptr(w_qabs), c_q.shape[-1], _ptr(w_uv),
                                                 _ptr(out), first_frame, n_frames, _stream(stream)),
              "vmla_chunk_attention_qlatent")

    def fold_output_weights(self, w_o, w_uv, w_fold, stream=None):
        """w_fold [d_out][n_h * d_c] = W_O,h W_uv,h side by side."""
        check(lib().vmla_fold_output_weights(ctypes.byref(self.cfg), _ptr(w_o), _ptr(w_uv), _ptr(w_fold),
                                             w_fold.shape[0], _stream(stream)), "vmla_fold_output_weights")

    def attention_folded(self, layer, q, w_uk, w_fold, out, first_frame, n_frames, stream=None):
        """Absorbed chunk attention with W_uv folded into the output mixer: out [B][rows][d_out] fp32."""
        check(lib().vmla_chunk_attention_folded(self._h, layer, _ptr(q), _ptr(w_uk), _ptr(w_fold), w_fold.shape[0],
                                                _ptr(out), first_frame, n_frames, _stream(stream)),
              "vmla_chunk_attention_folded")

    def set_append_tiling(self, n_split: int = 0, row_tiles: int = 0, max_ctas: int = 0):
        """Column parts, 128-row tiles per work item (0: chosen per call) and grid cap (0: one CTA
        per SM) of the append kernel."""
        check(lib().vmla_set_append_tiling(self._h, n_split, row_tiles, max_ctas), "vmla_set_append_tiling")

    def profile(self, enable: bool = True):
        """vmla_profile_enable: CUDA-event timing of every stage of the following calls."""
        check(lib().vmla_profile_enable(self._h, int(enable)), "vmla_profile_enable")

    def profile_read(self, stage) -> tuple:
        """vmla_profile_read: (summed milliseconds, launches) of a stage, by name or number."""
        st = STAGES[stage] if isinstance(stage, str) else stage
        ms, n = c_double(), c_int()
        check(lib().vmla_profile_read(self._h, st, ctypes.byref(ms), ctypes.byref(n)), "vmla_profile_read")
        return ms.value, n.value


def selftest_exp2(x, y, stream=None):
    """y = the kernels' polynomial 2^x (fp32 device tensors, even length)."""
    check(lib().vmla_selftest_exp2(x.data_ptr(), y.data_ptr(), x.numel(), _stream(stream)), "vmla_selftest_exp2")


def selftest_wait_timeout(limit_ns: int, stream=None):
    """vmla_selftest_wait_timeout: a kernel waiting on a flag nothing sets must give up and report."""
    check(lib().vmla_selftest_wait_timeout(limit_ns, _stream(stream)), "vmla_selftest_wait_timeout")
