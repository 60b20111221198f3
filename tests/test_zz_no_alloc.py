"""The allocation-free entry point (vmla_chunk_attention_noalloc) against the
workspace entry point (vmla_chunk_attention), through the C ABI.

It is meant for callers that cannot allocate device memory (a plugin handed
only its inputs and outputs, or a loop where cudaMalloc is not allowed); its
scratch is a fixed array inside the library.  This file is collected last so
that a run stopping at its first failure has already run every other test.
"""
import ctypes

import pytest

from latent_kv_attention_down_b200 import api, synth
from tests.harness import Rollout, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _noalloc(ro, q, out, first, n, frames):
    import torch
    w = ro.wd[0]
    return api.lib().vmla_chunk_attention_noalloc(
        ctypes.byref(ro.cfg), 0, ro.m.ckv.data_ptr(), ro.m.kr.data_ptr(), frames, q.data_ptr(), w[1].data_ptr(),
        w[2].data_ptr(), out.data_ptr(), first, n, torch.cuda.current_stream().cuda_stream)


SPLIT_64 = synth.WAN_SMALL.replace(name="wan_small_r64", d_nope=64, d_rope=64, rope_pairs=(12, 10, 10))
SPLIT_96 = synth.WAN_SMALL.replace(name="wan_small_r96", d_nope=32, d_rope=96, rope_pairs=(16, 16, 16))


@pytest.mark.parametrize("dims", [synth.WAN_SMALL, synth.WAN, SPLIT_64, SPLIT_96], ids=lambda d: d.name)
def test_noalloc_matches_workspace_entry_point_twice(dims):
    """Both entry points launch the same kernels with the same arguments, so the outputs must be
    equal bit for bit, on two calls in a row (the second one reuses the array as the first left
    it), on the small grid and on the full Wan-1.3B layer (27.3 MB of scratch)."""
    import torch
    d = dims
    ro = Rollout(d)
    for c in range(8):  # 24 frames through the 21-frame ring
        ro.append_chunk(0, c)
    q = to_dev(synth.queries(d, 0, 7), d)
    shape = (1, d.n_queries, d.n_heads * d.d_head)
    ref = torch.full(shape, float("nan"), dtype=torch.float32, device="cuda")
    ro.m.attention(0, q, ro.wd[0][1], ro.wd[0][2], ref, 21, 3, api.DESIGN_ABSORBED)
    assert ro.m.device_status()[0] == 0
    assert torch.isfinite(ref).all()
    for call in range(2):
        out = torch.full(shape, float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc(ro, q, out, 21, 3, 24) == 0
        assert ro.m.device_status()[0] == 0
        assert torch.equal(out, ref), f"no-alloc call {call} differs from the workspace entry point"


def test_noalloc_rejects_calls_beyond_its_array():
    import torch
    d = synth.WAN.replace(name="wan_b2", batch=2)  # 2 x 25.2 MB of absorbed queries > 32 MiB
    cfg = api.config_from_dims(d)
    dummy = torch.empty(256, dtype=torch.uint8, device="cuda")
    p = dummy.data_ptr()
    st = api.lib().vmla_chunk_attention_noalloc(ctypes.byref(cfg), 0, p, p, 21, p, p, p, p, 18, 3,
                                                torch.cuda.current_stream().cuda_stream)
    assert st == 3  # VMLA_ERR_OUT_OF_RANGE, nothing enqueued
