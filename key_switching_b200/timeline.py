"""Per-CTA timeline of one key switch (measurement tool).

    python -m key_switching_b200.build --timeline
    python -m key_switching_b200.timeline [--workload rot1_n16] [--steps 60] [--no-graph] [--json FILE]

Runs `steps` key switches of a single-ciphertext workload (each a replay of a
CUDA graph of pc_keyswitch, inputs rotated over sets larger than L2, as the
bench times them) with the library built with the per-CTA timeline, then
prints, for the last key switch, when each kernel's CTAs started and ended
(microseconds from its first CTA) and how many CTAs of each kernel were
resident over time.  The timestamps are the GPU's global nanosecond timer,
read by thread 0 of each CTA at entry and exit.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import sys


def summarize(tl, roles, bin_us: float = 4.0):
    """(per-role summary dict, occupancy rows) from a timeline array
    [roles][CTAs][3] of (start ns, end ns, SM)."""
    import numpy as np
    used = [r for r in range(len(roles)) if (tl[r][:, 0] > 0).any()]
    if not used:
        return {}, []
    t0 = min(int(tl[r][tl[r][:, 0] > 0][:, 0].min()) for r in used)
    summ, spans = {}, {}
    for r in used:
        m = tl[r][:, 0] > 0
        st = (tl[r][m][:, 0].astype(np.int64) - t0) / 1e3
        en = (tl[r][m][:, 1].astype(np.int64) - t0) / 1e3
        d = en - st
        spans[r] = (st, en)
        summ[roles[r]] = {"ctas": int(m.sum()), "sms": int(len(set(tl[r][m][:, 2].tolist()))),
                          "first_start_us": round(float(st.min()), 2), "last_start_us": round(float(st.max()), 2),
                          "first_end_us": round(float(en.min()), 2), "last_end_us": round(float(en.max()), 2),
                          "cta_us_median": round(float(np.median(d)), 2), "cta_us_min": round(float(d.min()), 2),
                          "cta_us_max": round(float(d.max()), 2)}
    end = max(float(en.max()) for _, en in spans.values())
    rows = []
    for k in range(int(math.ceil(end / bin_us)) + 1):
        t = k * bin_us
        rows.append((t, {roles[r]: int(((st <= t) & (en > t)).sum()) for r, (st, en) in spans.items()}))
    return summ, rows


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--workload", default="rot1_n16")
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--no-graph", action="store_true", help="call the library each step instead of replaying a graph")
    ap.add_argument("--bin-us", type=float, default=4.0, help="time step of the residency table")
    ap.add_argument("--json", default=None, help="also write the summary and the table to this file")
    args = ap.parse_args(argv)

    import numpy as np
    import torch

    os.environ.setdefault("PC_TIMELINE", "1")  # before the binding is first imported
    from . import pc, synth
    if not pc.TIMELINE:
        sys.exit("set PC_TIMELINE=1 before the binding is imported")
    wl = synth.WORKLOADS[args.workload]
    if wl.op != "keyswitch" or wl.n_ct != 1:
        sys.exit("a single-ciphertext key-switch workload is expected")
    q, p = pc.chain(wl.logN, wl.bits, wl.L, wl.alpha)
    ctx = pc.Context(wl.logN, q, p, device=0)
    N, L = wl.N, wl.L
    l = max(wl.levels) if wl.levels else L
    ctx.ensure_workspace(l, 1)
    prim = q + p
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint32).view(np.int32)).cuda()
    per_set = 2 * l * N * 4 + wl.dnum * (L + wl.alpha) * N * 4
    nsets = max(2, math.ceil(2 * 126e6 / per_set))
    sets = []
    for s in range(nsets):
        b = np.stack([synth.uniform_residues(prim, N, 1000 * s + 1, 0xB, j) for j in range(wl.dnum)])
        key = pc.KSK(synth.chacha_seed(1000 * s + 1, 0), dev(b), None)
        ct = dev(np.stack([synth.uniform_residues(q[:l], N, 50 + s, 0, 0, h) for h in range(2)]))
        sets.append((ct, key))
    out = torch.empty((2, l, N), dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()

    def run(ct, key, st):
        ctx.keyswitch(ct[0], ct[1], l, key, out[0], out[1], st)
    graphs = None if args.no_graph else [ctx.capture(lambda st, ct=ct, key=key: run(ct, key, st), keep=(ct, key))
                                         for ct, key in sets]
    for k in range(args.steps):
        if graphs:
            graphs[k % nsets].launch(stream)
        else:
            run(*sets[k % nsets], stream)
    torch.cuda.synchronize()
    summ, rows = summarize(ctx.timeline_read(), pc.TL_ROLES, args.bin_us)
    names = list(summ)
    print(f"# per-CTA timeline, {args.workload} (N=2^{wl.logN}, l={l}), "
          f"{'graph replay' if graphs else 'library calls'}, last of {args.steps} key switches")
    print("| kernel | CTAs | SMs | first start | last start | first end | last end | CTA median / min / max (us) |")
    print("|---|---|---|---|---|---|---|---|")
    for n, d in summ.items():
        print(f"| {n} | {d['ctas']} | {d['sms']} | {d['first_start_us']} | {d['last_start_us']} | "
              f"{d['first_end_us']} | {d['last_end_us']} | {d['cta_us_median']} / {d['cta_us_min']} / "
              f"{d['cta_us_max']} |")
    print()
    print("| t (us) | " + " | ".join(names) + " |")
    print("|---" * (len(names) + 1) + "|")
    for t, c in rows:
        print(f"| {t:g} | " + " | ".join(str(c.get(n, 0)) for n in names) + " |")
    if args.json:
        with open(args.json, "w") as f:
            json.dump({"workload": args.workload, "graph": graphs is not None, "summary": summ,
                       "resident": [{"t_us": t, **c} for t, c in rows]}, f, indent=1)
    for g in graphs or []:
        g.close()


if __name__ == "__main__":
    main()
