"""Per-configuration parity report: the CUDA path against the fp64 oracle on the five
benchmark configurations, one JSON line each (test infrastructure; needs a B200).

    python -m tests.parity_report

For each configuration it runs the library once through its public API on the full-size
seeded inputs and compares with the oracle on the samples the parity tests use:
  tiny     every head;
  gpt2     8 seeded heads (whole heads);
  causal   8 seeded heads, the last head of each batch entry among them;
  bwd      the same heads' dQ, dK, dV;
  long     2 seeded heads, 920 query rows each (the first and last 160, rows 4000-4199 around
           the band's first full width, 400 seeded ones).
It prints the O max-abs and mean-abs errors, the logsumexp max-abs error (gradients: relative
L2 of each), whether each is within the tolerance, and the oracle's wall time for its sample
(with the host's core count).
"""

from __future__ import annotations

import json
import os
import time

import numpy as np
import torch

from oracle import attention as orc
from synthetic import WORKLOADS, head_subset, make_grad_output, make_inputs
from tests.parity import GRAD_REL_L2, L_MAX_ABS, O_MAX_ABS, O_MEAN_ABS, forward_errors, rel_l2


def _heads(wl, n):
    return sorted(set(head_subset(wl, n)) | {(b + 1) * wl.H - 1 for b in range(wl.B)})


def _fwd_line(name, wl, o, lse, o_ref, l_ref, secs, sample):
    err = forward_errors(o, lse, o_ref, l_ref)
    ok = err["o_max"] <= O_MAX_ABS and err["o_mean"] <= O_MEAN_ABS and err["l_max"] <= L_MAX_ABS
    return {"config": name, "sample": sample, **{k: float(f"{v:.3e}") for k, v in err.items()},
            "within_tolerance": bool(ok), "oracle_s": round(secs, 2), "cores": os.cpu_count()}


def main():
    import exact_io_aware_77_b200 as fa
    fa.load()
    out = []
    for name in ("tiny", "gpt2", "causal"):
        wl = WORKLOADS[name]
        q, k, v = make_inputs(wl)
        o, lse = fa.forward(q.cuda(), k.cuda(), v.cuda(), wl.scale, wl.causal, wl.window)
        assert fa.check_status() == 0
        o, lse = o.cpu(), lse.cpu()
        heads = list(range(wl.BH)) if name == "tiny" else _heads(wl, 7)
        sel = lambda x: x.reshape(wl.BH, wl.N, -1)[heads]
        t0 = time.time()
        o_ref, l_ref = orc.attention_forward(sel(q), sel(k), sel(v), wl.scale, wl.causal, wl.window)
        secs = time.time() - t0
        out.append(_fwd_line(name, wl, sel(o), lse.reshape(wl.BH, wl.N)[heads], o_ref, l_ref, secs,
                             f"heads {heads}"))

    wl = WORKLOADS["bwd"]
    q, k, v = make_inputs(wl)
    do = make_grad_output(wl)
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    o, lse = fa.forward(qd, kd, vd, wl.scale, wl.causal, wl.window)
    grads = fa.backward(qd, kd, vd, o, lse, dod, wl.scale, wl.causal, wl.window)
    assert fa.check_status() == 0
    heads = _heads(wl, 7)
    sel = lambda x: x.reshape(wl.BH, wl.N, wl.d)[heads]
    t0 = time.time()
    refs = orc.attention_backward(sel(q), sel(k), sel(v), sel(do), wl.scale, wl.causal, wl.window)
    secs = time.time() - t0
    errs = {n: rel_l2(sel(g.cpu()), r) for n, g, r in zip(("dq", "dk", "dv"), grads, refs)}
    out.append({"config": "bwd", "sample": f"heads {heads}",
                **{f"{n}_rel_l2": float(f"{e:.3e}") for n, e in errs.items()},
                "within_tolerance": all(e <= GRAD_REL_L2 for e in errs.values()), "oracle_s": round(secs, 2),
                "cores": os.cpu_count()})

    wl = WORKLOADS["long"]
    q, k, v = make_inputs(wl)
    o, lse = fa.forward(q.cuda(), k.cuda(), v.cuda(), wl.scale, wl.causal, wl.window)
    assert fa.check_status() == 0
    o, lse = o.cpu(), lse.cpu()
    rng = np.random.default_rng(wl.seed)
    rows = np.unique(np.concatenate([np.arange(0, 160), np.arange(4000, 4200), np.arange(wl.N - 160, wl.N),
                                     rng.choice(wl.N, 400, replace=False)]))
    heads = head_subset(wl, wl.oracle_heads)
    o_s, l_s, o_r, l_r, secs = [], [], [], [], 0.0
    for h in heads:
        qh, kh, vh = (x.reshape(wl.BH, wl.N, wl.d)[h] for x in (q, k, v))
        t0 = time.time()
        a, b = orc.attention_forward_rows(qh, kh, vh, wl.scale, wl.causal, wl.window, rows=rows)
        secs += time.time() - t0
        o_r.append(a)
        l_r.append(b)
        o_s.append(o.reshape(wl.BH, wl.N, wl.d)[h][rows])
        l_s.append(lse.reshape(wl.BH, wl.N)[h][rows])
    out.append(_fwd_line("long", wl, torch.stack(o_s), torch.stack(l_s), np.stack(o_r), np.stack(l_r), secs,
                         f"heads {heads}, {len(rows)} rows each"))
    for line in out:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
