"""Launch one kernel of the chunk-attention path a few times, for a profiler.

    python -m latent_kv_attention_down_b200.profile_kernels {absorbed,recon,reconstruct,append1,append8}

Fills a 21-frame window of two Wan-1.3B-shaped layers (30x52 grid, 4680 queries per chunk) from
seeded synthetic frames, then makes four calls of the chosen kind: absorbed attention,
reconstruct-once attention, reconstruct-in-tile attention, or the cache append at batch 1 / 8.
Each run exits non-zero if the library reports a device-side error.
"""
from __future__ import annotations

import argparse
import sys


def main(argv=None) -> int:
    import torch
    from latent_kv_attention_down_b200 import api, synth
    ap = argparse.ArgumentParser()
    ap.add_argument("what", choices=["absorbed", "recon", "reconstruct", "append1", "append8"])
    ap.add_argument("--calls", type=int, default=4)
    args = ap.parse_args(argv)
    bf = torch.bfloat16
    batch = 8 if args.what == "append8" else 1
    d = synth.WAN.replace(batch=batch)
    design = {"absorbed": api.DESIGN_ABSORBED, "recon": api.DESIGN_RECON_ONCE,
              "reconstruct": api.DESIGN_RECONSTRUCT}.get(args.what, api.DESIGN_ABSORBED)
    m = api.LatentKVAttention(api.config_from_dims(d, layers=2)).allocate(design=design)
    pool = synth.FramePool(d)
    xp = torch.from_numpy(pool.x).cuda().to(bf)
    qp = torch.from_numpy(pool.q).cuda().to(bf)
    w = synth.weights(d, 0)
    W = [torch.from_numpy(a).cuda().to(bf) for a in (w.w_down, w.w_uk, w.w_uv)]
    out = torch.empty(batch, d.n_queries, d.n_heads * d.d_head, device="cuda")
    for layer in range(2):
        for c in range(7):
            m.append(layer, pool.activations(layer, c, 0, pool=xp), W[0], 3 * c, 3)
    q = [pool.queries(layer, 6, 0, pool=qp) for layer in range(2)]
    x = [pool.activations(layer, 6, 1, pool=xp) for layer in range(2)]
    for i in range(args.calls):
        if args.what.startswith("append"):
            m.append(i % 2, x[i % 2], W[0], 18, 3)
        else:
            m.attention(i % 2, q[i % 2], W[1], W[2], out, 18, 3, design)
    torch.cuda.synchronize()
    st, flags = m.device_status()
    print(args.what, "device status", st, hex(flags))
    return 0 if st == 0 else 1


if __name__ == "__main__":
    sys.exit(main())
