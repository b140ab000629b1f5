"""Miss rates of the shared LRU, a layer-oriented static split and prefill-time
hot placement, with the offline optimum as a bound, on the 40-layer NVFP4
decode trace (L = 40, E = 256, top-6, Zipf(1.0) routing with 10 % of the
popularity ranks reshuffled every 32 steps), at several cache capacities.

Routing comes from this library's GPU router (``moe_router_topk``) on the
seeded synthetic inputs of the trace workload; the policies are replayed on
the host (``policy.py``).  The prefill used for hot placement is a
1024-token prompt routed with the first drift epoch's router bias.

    python -m expert_cached_sparse_b200.policy_study [--steps 256] [--capacities 256,512,1024,2048]
"""
from __future__ import annotations

import argparse
import json


def route_trace(cfg, steps: int, prefill_tokens: int, device):
    """-> (decode trace [(layer, ids)] in step-major order, prefill trace)."""
    import numpy as np
    import torch

    from . import api as A
    from . import workloads as W

    def to_dev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(torch.bfloat16)

    E, k, H = cfg.experts, cfg.top_k, cfg.hidden
    per_layer = {}
    prefill = []
    for l in range(cfg.layers):
        wg = to_dev(W.gen_wg(cfg, 0, l))
        epochs = (steps + cfg.drift_every - 1) // cfg.drift_every if cfg.drift_every else 1
        rows = []
        for ep in range(epochs + 1):
            bias = torch.from_numpy(W.gen_bias(cfg, 0, l, ep)).to(device)
            if ep == epochs:   # the prefill prompt, routed with the first epoch's bias
                n = prefill_tokens
                bias = torch.from_numpy(W.gen_bias(cfg, 0, l, 0)).to(device)
                x = to_dev(W.gen_x(cfg, 0, n, "policy-prefill", l))
            else:
                s0 = ep * cfg.drift_every if cfg.drift_every else 0
                n = min(steps, s0 + (cfg.drift_every or steps)) - s0
                x = to_dev(np.concatenate([W.gen_x(cfg, 0, 1, "policy-decode", l, s) for s in range(s0, s0 + n)]))
            logits = torch.empty(n, E, dtype=torch.float32, device=device)
            idx = torch.empty(n, k, dtype=torch.int32, device=device)
            w = torch.empty(n, k, dtype=torch.float32, device=device)
            A.moe_router_topk(x, wg, bias, n, H, E, k, logits, idx, w)
            torch.cuda.synchronize()
            ids = idx.cpu().numpy()
            if ep == epochs:
                prefill += [(l, ids)]
            else:
                rows.append(ids)
        per_layer[l] = np.concatenate(rows)[:steps]
    decode = [(l, per_layer[l][s]) for s in range(steps) for l in range(cfg.layers)]
    return decode, prefill


def main(argv=None) -> int:
    import torch

    from . import policy as P
    from . import workloads as W

    p = argparse.ArgumentParser()
    p.add_argument("--steps", type=int, default=256)
    p.add_argument("--prefill-tokens", type=int, default=1024)
    p.add_argument("--capacities", default="256,512,1024,2048")
    args = p.parse_args(argv)
    cfg = W.TRACE40
    decode, prefill = route_trace(cfg, args.steps, args.prefill_tokens, torch.device("cuda", 0))
    out = {"workload": "40-layer trace: E=256, top-6, Zipf(1.0), 10% rank drift every 32 steps, "
                       f"{args.steps} one-token steps", "reads_per_step": None, "capacity": {}}
    for c in (int(v) for v in args.capacities.split(",")):
        res = {"shared_lru": P.replay(P.SharedLru(c), decode),
               "static_layer_split": P.replay(P.StaticPlacement(P.layer_split(cfg.layers, cfg.experts, c)), decode),
               "prefill_hot": P.replay(P.StaticPlacement(P.prefill_hot(prefill, c)), decode),
               "belady_bound": P.belady(decode, c)}
        out["capacity"][c] = {k: round(v["miss_rate"], 4) for k, v in res.items()}
        out["reads_per_step"] = res["shared_lru"]["reads"] / args.steps
    print(json.dumps(out), flush=True)
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
