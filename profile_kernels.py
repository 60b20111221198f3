"""Launch one kernel of the chunk-attention path a few times, for a profiler.

    python profile_kernels.py \
        {absorbed,recon,reconstruct,append1,append8,step8,folded,qlatent}

Fills a 21-frame window of two Wan-1.3B-shaped layers (30x52 grid, 4680 queries per chunk) from
seeded synthetic frames, then makes four calls of the chosen kind: absorbed attention,
reconstruct-once attention, reconstruct-in-tile attention, the cache append at batch 1 / 8, a
whole chunk step (append, RoPE, q-absorb, attention) at batch 8, absorbed attention with the
folded output mixer, or absorbed attention fed from the query latent.
Each run exits non-zero if the library reports a device-side error.
"""
from __future__ import annotations

import argparse
import sys


def main(argv=None) -> int:
    import torch
    from latent_kv_attention_down_b200 import api, synth
    ap = argparse.ArgumentParser()
    ap.add_argument("what", choices=["absorbed", "recon", "reconstruct", "append1", "append8", "step8", "folded",
                                     "qlatent"])
    ap.add_argument("--calls", type=int, default=4)
    args = ap.parse_args(argv)
    bf = torch.bfloat16
    batch = 8 if args.what in ("append8", "step8") else 1
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
    extra = None
    if args.what == "folded":
        extra = torch.empty(d.d_model, d.n_heads * d.d_latent, dtype=bf, device="cuda")
        m.fold_output_weights(torch.from_numpy(w.w_o).cuda().to(bf), W[2], extra)
        out = torch.empty(batch, d.n_queries, d.d_model, device="cuda")
    elif args.what == "qlatent":
        w_uq, w_qr = synth.query_latent_weights(d, 0)
        extra = torch.empty(d.n_heads, d.d_latent + d.d_rope, d.d_q, dtype=bf, device="cuda")
        m.fold_query_weights(torch.from_numpy(w_uq).cuda().to(bf), torch.from_numpy(w_qr).cuda().to(bf), W[1], extra)
        cq = torch.from_numpy(synth.query_latents(d, 0, 6)).cuda().to(bf)
    for i in range(args.calls):
        if args.what.startswith("append"):
            m.append(i % 2, x[i % 2], W[0], 18, 3)
        elif args.what == "step8":
            m.append(i % 2, x[i % 2], W[0], 18, 3)
            m.attention(i % 2, q[i % 2], W[1], W[2], out, 18, 3, design)
        elif args.what == "folded":
            m.attention_folded(i % 2, q[i % 2], W[1], extra, out, 18, 3)
        elif args.what == "qlatent":
            m.attention_qlatent(i % 2, cq, extra, W[2], out, 18, 3)
        else:
            m.attention(i % 2, q[i % 2], W[1], W[2], out, 18, 3, design)
    torch.cuda.synchronize()
    st, flags = m.device_status()
    print(args.what, "device status", st, hex(flags))
    return 0 if st == 0 else 1


if __name__ == "__main__":
    sys.exit(main())
