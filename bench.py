#!/usr/bin/env python
"""bench.py -- key-switches/s of CKKS hybrid key switching on B200.

Default workload (one step = one key switch, pc_keyswitch):
  N=2^16, L=24 ciphertext primes + alpha=4 special primes (31-bit), dnum=6,
  one ciphertext at the top level (l=24), rotation key whose uniform half is
  regenerated in-kernel from its ChaCha12 seed; inputs are seeded uniform
  residues, rotated over enough (ciphertext, key) sets that the step's inputs
  exceed the 126 MB L2.  Each step replays a CUDA graph of the call captured
  for its input set, except every 30th step, a direct call carrying per-kernel
  CUDA events (the live roofline); --no-graph calls the library every step.

Other workloads (--workload): relin_n12 (N=2^12 s^2 -> s key switch),
batch16_n16 (16 ciphertexts, 16 keys, one batched call), ntt_n16 (64 x 28-limb
forward + inverse NTTs), sweep_n17 (N=2^17, levels 40..1), rotate_n16 (one
rotation), hoisted8_n16 (8 rotations sharing one ModUp), relin_mul_n12 /
relin_mul_n16 (ciphertext product: tensor + relinearisation).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--keys regen|stored] [--no-graph] [--impl ours|reference]

Prints one JSON line (rank 0) with the roofline of the dominant kernel, the
oracle's single-core CPU baseline (single-GPU runs) and the end-to-end rate of
host-resident ciphertexts through pc_keyswitch_host.  Multi-GPU (torchrun):
every rank runs its own independent key switches (weak scaling, no data-path
collective); the time is the max over ranks.  --impl reference times the plain
CPU oracle on the host cores instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L2_BYTES = 126 * 2**20
# DRAM bytes (read + write) per launch of the roofline kernel, from one ncu
# capture of the current kernel (profiles/k_inner_keyswitch_n16.md, cold
# cache); None when the kernel has changed since the counters were taken.
KERNEL_TRAFFIC = {("rot1_n16", "inner_chacha"): 104.93e6 + 5.13e6}
# A Shoup modular multiply is IMAD.HI + 2 IMAD on the 16-lane-per-partition
# multiply-add pipe, and the high-half multiply occupies two issue slots:
# 4 slots of 64 lanes/SM/clock (measured by pc_microbench kind 0 at 4.57 T/s)
MODMUL_IMAD = 4
IMAD_PER_SM_CLK = 64  # 32-bit IMAD lanes per SM per clock
SMS = 148
# One ChaCha12 block: 6 double rounds x 8 quarter rounds x (4 add, 4 xor,
# 4 rotate) + 16 feed-forward adds = 592 32-bit lane operations; the xors and
# rotates (384) run on the ALU pipe, the adds on either pipe.
CHACHA_OPS = 6 * 8 * 12 + 16
# Integer issue ceiling: one warp instruction per partition per clock,
# 4 partitions x 32 lanes = 128 lane operations per SM per clock (the ALU and
# multiply-add pipes at 64 lanes each, both busy).
ISSUE_LANES_PER_SM_CLK = 128


# ----------------------------------------------------------------- workloads

def workload_counts(logN: int, L: int, alpha: int, l: int, regen: bool = True):
    """Algorithmic work of one key switch at level l (spec v1 dataflow):
    modular multiplies (butterflies, conversions, products), HBM bytes of the
    inputs and outputs that must move, and ChaCha12 blocks."""
    N = 1 << logN
    beta = -(-l // alpha)
    ll = l + alpha
    half_logN = N // 2 * logN          # butterflies of one limb NTT
    d = [min(alpha, l - j * alpha) for j in range(beta)]
    intt_c1 = l * half_logN + l * N     # + one scale multiply per coefficient
    modup_conv = sum(dj * (ll - dj) * N for dj in d)
    modup_ntt = sum((ll - dj) for dj in d) * half_logN
    inner = 2 * beta * ll * N
    md_intt = 2 * alpha * half_logN + 2 * alpha * N
    md_conv = 2 * alpha * l * N
    md_ntt = 2 * l * half_logN
    md_scale = 2 * l * N
    modmuls = intt_c1 + modup_conv + modup_ntt + inner + md_intt + md_conv + md_ntt + md_scale
    key_bytes = beta * ll * N * 4 * (1 if regen else 2)
    bytes_ = 2 * l * N * 4 + key_bytes + 2 * l * N * 4
    blocks = beta * ll * N // 8 if regen else 0
    return {"modmuls": modmuls, "bytes": bytes_, "chacha_blocks": blocks}


def op_counts(wl, l: int, regen: bool = True):
    """Work of one step's unit of the workload's operation at level l: a key
    switch or rotation (the automorphism is a permutation: no arithmetic), a
    relinearisation (key switch + 4 slot products per coefficient, reading two
    ciphertexts), or n_rot hoisted rotations (one ModUp, n_rot inner products
    and ModDowns)."""
    ks = workload_counts(wl.logN, wl.L, wl.alpha, l, regen)
    N = 1 << wl.logN
    if wl.op == "relin":
        return {"modmuls": ks["modmuls"] + 4 * l * N, "bytes": ks["bytes"] + 2 * l * N * 4,
                "chacha_blocks": ks["chacha_blocks"]}
    if wl.op == "hoisted":
        st = stage_modmuls(wl.logN, wl.L, wl.alpha, l)
        up = st["intt_row_c1"] + st["modup_col"]
        n = wl.n_rot
        key_bytes = ks["bytes"] - 4 * l * N * 4
        return {"modmuls": up + n * (ks["modmuls"] - up), "bytes": 2 * l * N * 4 + n * (key_bytes + 2 * l * N * 4),
                "chacha_blocks": n * ks["chacha_blocks"]}
    return ks


def stage_modmuls(logN: int, L: int, alpha: int, l: int):
    """Modular multiplies done by each profiled stage (kernel) of one key switch."""
    N = 1 << logN
    logC = min(8, logN - 4)
    logR = logN - logC
    beta = -(-l // alpha)
    ll = l + alpha
    d = [min(alpha, l - j * alpha) for j in range(beta)]
    ntarg = sum(ll - dj for dj in d)
    return {
        "intt_row_c1": l * (N // 2) * logC,
        "modup_col": l * (N // 2) * logR + l * N
        + sum(dj * (ll - dj) for dj in d) * N + ntarg * (N // 2) * logR,
        "inner_chacha": ntarg * (N // 2) * logC + 2 * beta * ll * N + 2 * alpha * (N // 2) * logC,
        "moddown_col": 2 * alpha * (N // 2) * logR + 2 * alpha * N
        + 2 * alpha * l * N + 2 * l * (N // 2) * logR,
        "moddown_finish": 2 * l * (N // 2) * logC + 2 * l * N,
    }


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.device = device
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.device), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for ln in open(self.path).read().splitlines():
            f = [x.strip() for x in ln.split(",")]
            if len(f) >= 9:
                rows.append(f)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------ distributed

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x: float, dist=None, device="cpu") -> float:
    """The largest value of x over all ranks (every rank gets it); x itself
    without a process group.  Used for the device-timed region, so the
    slowest rank sets the job's time."""
    if dist is None:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank_step: float, steps: int, world: int, max_ms: float) -> float:
    """Units per second of the whole job: every rank processes its own units
    (weak scaling), the time is the slowest rank's."""
    return units_per_rank_step * steps * world / (max_ms * 1e-3)


# --------------------------------------------------------------- our arm

def run_ours(args):
    import numpy as np
    import torch
    import datetime

    from key_switching_b200 import pc, synth

    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    wl = synth.WORKLOADS[args.workload]
    q, p = pc.chain(wl.logN, wl.bits, wl.L, wl.alpha)
    ctx = pc.Context(wl.logN, q, p, device=local)
    N, L, A = wl.N, wl.L, wl.alpha
    regen = args.keys == "regen"
    prim = q + p
    stream = torch.cuda.current_stream()
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint32).view(np.int32)).cuda()

    def make_key(seed_id):
        b = np.stack([synth.uniform_residues(prim, N, seed_id, 0xB, j) for j in range(wl.dnum)])
        a = None
        if not regen:
            a = dev(np.stack([synth.uniform_residues(prim, N, seed_id, 0xA, j) for j in range(wl.dnum)]))
        return pc.KSK(synth.chacha_seed(seed_id, rank), dev(b), a)

    launches_per_step = 5
    graphs = None
    PROF_EVERY = 30  # sampled steps carry per-kernel events; the rest run uninstrumented
    if args.workload == "ntt_n16":
        unit, metric = "limb-NTTs/s", "forward+inverse negacyclic NTT throughput at N=2^16 (1 B200)"
        NPL = L + A
        per_set = wl.n_ct * NPL * N * 4
        nsets = max(2, math.ceil(2 * L2_BYTES / per_set))
        sets = [dev(synth.uniform_residues_batch(prim, N, wl.n_ct, 40 + s, rank)) for s in range(nsets)]
        units_per_step = 2 * wl.n_ct * NPL

        def step(k):
            x = sets[k % nsets]
            ctx.ntt_fwd(x, 0, NPL, wl.n_ct, stream)
            ctx.ntt_inv(x, 0, NPL, wl.n_ct, stream)
        launches_per_step = 4
        levels = [L]
        work = None
    else:
        unit, metric = "key-switches/s", "key-switches/s at N=2^16 (1 B200); achieved HBM GB/s and % of roofline"
        if args.workload == "sweep_n17":
            metric = "key-switches/s at N=2^17 level sweep 40..1 (1 B200)"
        if wl.op in ("rotate", "hoisted"):
            unit = "rotations/s"
            metric = (f"rotations/s at N=2^{wl.logN} ({'single' if wl.op == 'rotate' else f'{wl.n_rot} hoisted'}"
                      " rotation(s) per ciphertext; 1 B200)")
        elif wl.op == "relin":
            unit = "relinearisations/s"
            metric = f"ciphertext products (tensor + relinearisation) per second at N=2^{wl.logN} (1 B200)"
        levels = list(wl.levels) if wl.levels else [L]
        B = wl.n_ct
        nk = wl.n_rot if wl.op == "hoisted" else B  # keys per step
        ctx.ensure_workspace(max(levels), max(B, min(wl.n_rot, 16)) if wl.op == "hoisted" else B)
        per_set = (B * (2 * L * N * 4) * (2 if wl.op == "relin" else 1)
                   + nk * wl.dnum * (L + A) * N * 4 * (1 if regen else 2))
        nsets = max(2, math.ceil(2 * L2_BYTES / per_set)) if args.workload != "sweep_n17" else 1
        sets = []
        nct = B * (2 if wl.op == "relin" else 1)
        for s in range(nsets):
            keys = [make_key(1000 * s + k + 1) for k in range(nk)]
            ct = dev(np.stack([np.stack([synth.uniform_residues(q, N, 50 + s, rank, k, h) for h in range(2)])
                               for k in range(nct)]))
            sets.append((ct, keys))
        out = torch.empty((max(B, wl.n_rot), 2, L, N), dtype=torch.int32, device="cuda")
        units_per_step = (wl.n_rot if wl.op == "hoisted" else B) * len(levels)
        rot_gs = [pow(5, 1 << r, 2 * N) for r in range(wl.n_rot)]  # steps 1, 2, 4, ...

        def run_op(ct, keys, st):
            """One step's library calls on stream st."""
            for l in levels:
                if wl.op == "rotate":
                    ctx.rotate(ct[0, 0, :l], ct[0, 1, :l], l, rot_gs[0], keys[0], out[0, 0, :l], out[0, 1, :l], st)
                elif wl.op == "hoisted":
                    ctx.rotate_hoisted(ct[0, 0, :l], ct[0, 1, :l], l, rot_gs, keys, out[:, :, :l], st)
                elif wl.op == "relin":
                    ctx.relinearize(ct[0, :, :l], ct[1, :, :l], l, keys[0], out[0, :, :l], st)
                elif B == 1:
                    # level-l ciphertext = the first l limbs of each half
                    ctx.keyswitch(ct[0, 0, :l], ct[0, 1, :l], l, keys[0], out[0, 0, :l], out[0, 1, :l], st)
                else:
                    ctx.keyswitch_batch(ct, B, l, keys, out, st)

        # one CUDA graph of a step per input set (single-ciphertext workloads;
        # a level sweep is one graph of all its key switches)
        if not args.no_graph and B == 1:
            graphs = [ctx.capture(lambda st, ct=ct, keys=keys: run_op(ct, keys, st), keep=(ct, keys))
                      for ct, keys in sets]

        def step(k):
            # graph replay, except every PROF_EVERY-th step: a direct call that
            # carries the per-kernel events (the sampled roofline timing)
            if graphs is not None and k % PROF_EVERY:
                graphs[k % nsets].launch(stream)
                return
            ct, keys = sets[k % nsets]
            run_op(ct, keys, stream)
        # 6 launches per key switch (the inner product splits in two when the
        # ModDown branch overlaps), 5 in the instrumented (serial) calls
        launches_per_step = (5 if os.environ.get("PC_NO_OVERLAP") else 6) * len(levels)
        if wl.op == "hoisted":  # one ModUp (2), then per rotation 4 (3 when serial)
            launches_per_step = (2 + (3 if os.environ.get("PC_NO_OVERLAP") else 4) * wl.n_rot) * len(levels)
        work = [op_counts(wl, l, regen) for l in levels]

    # warm-up, then exactly K timed steps between barriers
    for k in range(args.warmup):
        step(k)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    prof = args.workload != "ntt_n16"
    if prof:
        # with graphs every direct call is a sampled one
        ctx.profile_begin(args.steps * len(levels), 1 if graphs is not None else PROF_EVERY)
    clocks = ClockSampler(local)
    clocks.start()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for k in range(args.steps):
        step(k)
    e1.record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    stage_ms, ncalls = ctx.profile_end() if prof else ({}, 0)
    ms = max_over_ranks(ms, dist, "cuda")
    value = whole_job_rate(units_per_step, args.steps, world, ms)

    res = {"metric": metric, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "u32", "data": "synthetic (seeded uniform residues, "
           "uniform key 'b' halves; ChaCha12 seeds)",
           "config": {"workload": f"{wl.name}: N=2^{wl.logN}, L={L}, alpha={A}, dnum={wl.dnum}, "
                      f"{wl.n_ct} ct/step, levels {levels[0]}..{levels[-1]}, key a-half "
                      f"{'regenerated in-kernel (ChaCha12)' if regen else 'stored in HBM'}",
                      "l2": f"inputs rotated over {nsets} sets of {per_set / 1e6:.1f} MB (> 126 MB L2)",
                      "parallelism": f"replicas x{world}",
                      "launch": f"CUDA graph replay (every {PROF_EVERY}th step a direct, instrumented call)"
                      if graphs is not None else "library calls"},
           "gpu_launches": launches_per_step * args.steps
           - (0 if (os.environ.get("PC_NO_OVERLAP") or not prof) else ncalls), "clocks": clk}

    if work is not None:
        mm = sum(w["modmuls"] for w in work)
        by = sum(w["bytes"] for w in work)
        sec_per_step = ms * 1e-3 / args.steps / world * world  # per rank
        sm_mhz = clk.get("sm_mhz") or 1965.0
        peak_derived = SMS * IMAD_PER_SM_CLK * 1965e6 / MODMUL_IMAD
        try:
            peak_meas = pc.microbench(0, 2048, local) if rank == 0 else None
        except Exception:
            peak_meas = None
        hbm = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))["hbm_gbs"] \
            if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")) else 6650.0
        t_roof = max(by / (hbm * 1e9), mm / peak_derived)
        res["step_roofline"] = {"modmuls_per_step": mm * wl.n_ct, "hbm_bytes_per_step": by * wl.n_ct,
                                "achieved_gbs": by * wl.n_ct / sec_per_step / 1e9,
                                "achieved_tmodmul_s": mm * wl.n_ct / sec_per_step / 1e12,
                                "t_roofline_us": t_roof * wl.n_ct * 1e6, "t_step_us": sec_per_step * 1e6,
                                "frac": t_roof * wl.n_ct / sec_per_step,
                                "modmul_peak_derived": peak_derived,
                                "modmul_peak_microbench": peak_meas, "hbm_peak_gbs": hbm}
        if stage_ms and ncalls:
            smm = {}
            for l in levels:
                for kname, v in stage_modmuls(wl.logN, L, A, l).items():
                    smm[kname] = smm.get(kname, 0) + v * wl.n_ct
            # integer lane operations per stage: 4 per modular multiply, 592
            # per ChaCha12 block (the inner-product stage regenerates a)
            blocks = sum(w["chacha_blocks"] for w in work) * wl.n_ct
            sops = {k: MODMUL_IMAD * v for k, v in smm.items()}
            sops["inner_chacha"] += CHACHA_OPS * blocks
            peak_ops = SMS * ISSUE_LANES_PER_SM_CLK * 1965e6
            tot = sum(stage_ms.values())
            top = max(stage_ms, key=stage_ms.get)
            per_launch_s = stage_ms[top] * 1e-3 / ncalls * len(levels)
            ach = sops[top] / per_launch_s
            res["roofline"] = {"bound": "alu", "kernel": top, "achieved": ach / 1e12,
                               "peak": peak_ops / 1e12, "unit": "Tintop/s",
                               "frac": ach / peak_ops,
                               "traffic": KERNEL_TRAFFIC.get((args.workload, top)) if regen else None,
                               "share": stage_ms[top] / tot if tot else None,
                               "ops_per_launch": sops[top] / len(levels),
                               "modmul_frac": smm[top] / per_launch_s / peak_derived,
                               "peak_source": "derived: 148 SMs x 128 issued 32-bit lane ops/clk (4 partitions x "
                                              "32; ALU + multiply-add pipes) x 1965 MHz; ops = 4 per Shoup "
                                              "modular multiply + 592 per ChaCha12 block"}
            res["stage_ms_per_step"] = {k: v / ncalls * len(levels) for k, v in stage_ms.items()}
            res["stage_sampling"] = f"{ncalls} of {args.steps * len(levels)} calls instrumented (every {PROF_EVERY}th)"
        else:
            # no per-kernel events on this path (hoisted rotations): the whole step
            peak_ops = SMS * ISSUE_LANES_PER_SM_CLK * 1965e6
            ops = (MODMUL_IMAD * mm + CHACHA_OPS * sum(w["chacha_blocks"] for w in work)) * wl.n_ct
            ach = ops / sec_per_step
            res["roofline"] = {"bound": "alu", "kernel": "whole step", "achieved": ach / 1e12,
                               "peak": peak_ops / 1e12, "unit": "Tintop/s", "frac": ach / peak_ops,
                               "traffic": None,
                               "peak_source": "derived: 148 SMs x 128 issued 32-bit lane ops/clk x 1965 MHz; "
                                              "ops = 4 per Shoup modular multiply + 592 per ChaCha12 block"}

    # end-to-end: host buffers through the library's host-buffer call, every
    # step's copies inside the timed region (pipelined with the key switches)
    if not args.no_e2e and args.workload in ("rot1_n16", "relin_n12"):
        ct0, keys0 = sets[0]
        l = L
        ke = max(3, min(args.steps, 20))
        h_in = torch.empty((ke, 2, l, N), dtype=torch.int32).pin_memory()
        h_in.copy_(ct0[0].cpu().unsqueeze(0).expand(ke, 2, l, N))
        h_out = torch.empty((ke, 2, l, N), dtype=torch.int32).pin_memory()
        ctx.ensure_host_workspace(l)
        kk = [keys0[0]] * ke

        def e2e_run():
            ctx.keyswitch_host(h_in, ke, l, kk, h_out, stream)
        e2e_run()
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        e2e_run()
        f1.record(stream)
        torch.cuda.synchronize()
        ems = f0.elapsed_time(f1)
        ems = max_over_ranks(ems, dist, "cuda")
        res["e2e"] = {"value": whole_job_rate(1, ke, world, ems), "unit": unit,
                      "h2d_bytes_per_step": 2 * l * N * 4, "d2h_bytes_per_step": 2 * l * N * 4}

    # the oracle's CPU baseline: rank 0 of a single-GPU run only
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.workload in ("rot1_n16", "relin_n12"):
        res["cpu_baseline"] = cpu_baseline(wl, q, p, budget_s=args.cpu_budget)

    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


# ------------------------------------------------------------ oracle timing

def _oracle_inputs(wl, q, p):
    import numpy as np
    from key_switching_b200 import synth
    from oracle import oracle as O
    P = O.Params(wl.logN, q, p)
    prim = [P.prime(g) for g in range(P.L + P.alpha)]
    b = np.stack([synth.uniform_residues(prim, P.N, 1, 0xB, j) for j in range(P.dnum)])
    l = wl.L
    c0 = synth.uniform_residues(P.q[:l], P.N, 50, 0, 0, 0)
    c1 = synth.uniform_residues(P.q[:l], P.N, 50, 0, 0, 1)
    return O, P, b, c0, c1, l, synth.chacha_seed(1, 0)


def oracle_step(wl, O, P, b, c0, c1, l, seed):
    """One unit batch of the workload's operation on the oracle; returns the
    number of operations done (n_rot for hoisted rotations, else 1)."""
    from key_switching_b200 import synth
    if wl.op == "rotate":
        O.rotate(P, c0, c1, l, pow(5, 1, 2 * P.N), seed, b)
    elif wl.op == "hoisted":
        gs = [pow(5, 1 << r, 2 * P.N) for r in range(wl.n_rot)]
        O.rotate_hoisted(P, c0, c1, l, gs, [seed] * wl.n_rot, [b] * wl.n_rot)
        return wl.n_rot
    elif wl.op == "relin":
        y0 = synth.uniform_residues(P.q[:l], P.N, 51, 0, 0, 0)
        y1 = synth.uniform_residues(P.q[:l], P.N, 51, 0, 0, 1)
        O.relinearize(P, c0, c1, y0, y1, l, seed, b)
    else:
        O.keyswitch(P, c0, c1, l, seed, b)
    return 1


def _unit(wl):
    return {"rotate": "rotations/s", "hoisted": "rotations/s", "relin": "relinearisations/s"}.get(
        wl.op, "key-switches/s")


def cpu_baseline(wl, q, p, budget_s: float = 20.0):
    """The oracle as it stands, single-threaded, on a bounded sample: as many
    full operations of the workload as fit in about budget_s seconds."""
    O, P, b, c0, c1, l, seed = _oracle_inputs(wl, q, p)
    t0 = time.perf_counter()
    n = ops = 0
    while True:
        ops += oracle_step(wl, O, P, b, c0, c1, l, seed)
        n += 1
        if time.perf_counter() - t0 >= budget_s or n >= 50:
            break
    dt = time.perf_counter() - t0
    return {"value": ops / dt, "unit": _unit(wl), "cores": 1, "kind": "oracle",
            "sample": f"{n} full {wl.op} step(s) ({ops} operation(s)) of {wl.name} (l={l}) in {dt:.1f} s, "
                      "single thread"}


def run_reference(args):
    world, rank, local = dist_setup()
    if rank != 0:
        return
    from key_switching_b200 import pc, synth
    wl = synth.WORKLOADS[args.workload]
    q, p = pc.chain(wl.logN, wl.bits, wl.L, wl.alpha)
    O, P, b, c0, c1, l, seed = _oracle_inputs(wl, q, p)
    budget = args.cpu_budget * 6
    t0 = time.perf_counter()
    for _ in range(min(args.warmup, 1)):
        oracle_step(wl, O, P, b, c0, c1, l, seed)
    t_one = max(1e-3, time.perf_counter() - t0)
    steps = max(1, min(args.steps, int(budget / t_one)))
    t0 = time.perf_counter()
    ops = 0
    for _ in range(steps):
        ops += oracle_step(wl, O, P, b, c0, c1, l, seed)
    dt = time.perf_counter() - t0
    v = ops / dt
    unit = _unit(wl)
    metric = "key-switches/s at N=2^16 (1 B200); achieved HBM GB/s and % of roofline"
    if wl.op in ("rotate", "hoisted"):
        metric = (f"rotations/s at N=2^{wl.logN} ({'single' if wl.op == 'rotate' else f'{wl.n_rot} hoisted'}"
                  " rotation(s) per ciphertext; 1 B200)")
    elif wl.op == "relin":
        metric = f"ciphertext products (tensor + relinearisation) per second at N=2^{wl.logN} (1 B200)"
    elif wl.name == "sweep_n17":
        metric = "key-switches/s at N=2^17 level sweep 40..1 (1 B200)"
    res = {"impl": "reference", "metric": metric,
           "value": v, "unit": unit, "n_gpus": 1, "steps": steps, "warmup": min(args.warmup, 1),
           "ms_per_step": dt * 1e3 / steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
           "dtype": "u32", "data": "synthetic",
           "config": {"workload": f"{wl.name}: N=2^{wl.logN}, L={wl.L}, alpha={wl.alpha}, dnum={wl.dnum}, "
                      "1 ct/step at the top level, key a-half regenerated (ChaCha12)"},
           "cpu_baseline": {"value": v, "unit": unit, "cores": 1, "kind": "oracle",
                            "sample": f"{steps} of {args.steps} requested step(s), each one full {wl.op} "
                                      f"({ops} operation(s) in all), time-bounded, single thread"},
           "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="rot1_n16",
                    choices=["rot1_n16", "relin_n12", "batch16_n16", "ntt_n16", "sweep_n17", "rotate_n16",
                             "hoisted8_n16", "relin_mul_n12", "relin_mul_n16"])
    ap.add_argument("--keys", default="regen", choices=["regen", "stored"])
    ap.add_argument("--no-graph", action="store_true",
                    help="call pc_keyswitch every step instead of replaying a CUDA graph of it")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for cpu_baseline")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
