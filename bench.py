#!/usr/bin/env python
"""bench.py -- key-switches/s of CKKS hybrid key switching on B200.

Default workload (one step = one key switch, pc_keyswitch):
  N=2^16, L=24 ciphertext primes + alpha=4 special primes (31-bit), dnum=6,
  one ciphertext at the top level (l=24), rotation key whose uniform half is
  regenerated in-kernel from its ChaCha12 seed; inputs are seeded uniform
  residues, rotated over enough (ciphertext, key) sets that the step's inputs
  exceed the 126 MB L2.  Each timed step replays a CUDA graph of the call
  captured for its input set (--no-graph calls the library every step).
  After the timed region, a separate pass of at least 10 direct calls carries
  per-kernel CUDA events; their medians give the dominant kernel's roofline.

Other workloads (--workload): relin_n12 (N=2^12 s^2 -> s key switch),
batch16_n16 (16 ciphertexts, 16 keys, one batched call; split across the
ranks when run on several GPUs), ntt_n16 (64 x 28-limb forward + inverse
NTTs), sweep_n17 (N=2^17, levels 40..1), rotate_n16 (one rotation),
hoisted8_n16 (8 rotations sharing one ModUp), relin_mul_n12 / relin_mul_n16
(ciphertext product: tensor + relinearisation).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--keys regen|stored] [--no-graph] [--impl ours|reference]

Prints one JSON line (rank 0) with the roofline of the dominant kernel, the
oracle's CPU baseline on the host cores (single-GPU runs) and the end-to-end
rate of host-resident ciphertexts through pc_keyswitch_host.  With --gpus N
the script runs N ranks, one per GPU (started by torch.distributed.run, or by
itself when launched as one process): every rank runs its own key switches
(weak scaling, no data-path collective), except that the 16-pair batch is
split across the ranks (strong scaling); the time is the max over ranks.
--impl reference times the plain CPU oracle on the host cores instead (rank 0
only).
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
# DRAM bytes (read + write) of one launch of the roofline kernel, recorded
# from one ncu capture (--clock-control none, cold cache) of the kernel source
# whose hash is given; reported only while the kernel sources still hash to
# that value (otherwise the traffic is null: the counters are stale).
# (PC_NO_OVERLAP=1: the inner product as one launch over all l + alpha target
# limbs; one launch of a --set full capture -- counters-only captures of
# earlier, equivalent sources read the same 104.93 MB and wrote 2.3-6.3 MB, the
# rest of the accumulators still in L2 when the kernel ended)
KERNEL_TRAFFIC = {("rot1_n16", "inner_chacha"): (104.92672e6 + 6.181888e6, "47fe253dc7b4c677")}
KERNEL_SOURCES = ("kernels.cu", "ntt.cuh", "chacha.cuh", "modarith.cuh")


def kernel_source_hash() -> str:
    """First 16 hex digits of the SHA-256 of the kernel sources."""
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "key_switching_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


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
    if wl.op == "bsgs":
        # n1 - 1 hoisted baby rotations (one ModUp), n2 - 1 giant rotations,
        # n1 n2 diagonal products per half; bytes: ciphertext in and out, the
        # keys' b halves, the diagonals
        n1, n2 = wl.bsgs
        st = stage_modmuls(wl.logN, wl.L, wl.alpha, l)
        up = st["intt_row_c1"] + st["modup_col"]
        baby = (up + (n1 - 1) * (ks["modmuls"] - up)) if n1 > 1 else 0
        key_bytes = ks["bytes"] - 4 * l * N * 4
        return {"modmuls": baby + (n2 - 1) * ks["modmuls"] + 2 * n1 * n2 * l * N,
                "bytes": 4 * l * N * 4 + (n1 + n2 - 2) * key_bytes + n1 * n2 * l * N * 4,
                "chacha_blocks": (n1 + n2 - 2) * ks["chacha_blocks"]}
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
                                          "--format=csv,noheader,nounits", "-lms", "25"],
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


def shard(n_items: int, world: int, rank: int) -> range:
    """The contiguous share of n_items independent units that rank `rank` of
    `world` processes: sizes differ by at most one, every unit is in exactly
    one share."""
    lo = n_items * rank // world
    hi = n_items * (rank + 1) // world
    return range(lo, hi)


def rank_plan(workload: str, n_ct: int, world: int, rank: int, local: int):
    """What one rank runs: its device (the local rank's GPU) and the indices of
    the workload's (ciphertext, key) pairs it key-switches.  A batch of
    independent pairs is split across the ranks (strong scaling: the job's
    total is fixed); every other workload runs whole on every rank (weak
    scaling: replicas)."""
    if workload == "batch16_n16":
        return {"device": local, "items": shard(n_ct, world, rank), "scaling": "strong"}
    return {"device": local, "items": range(n_ct), "scaling": "weak"}


def launch_ranks(argv, n: int) -> int:
    """Re-run this script as n ranks on this node (one process per GPU) when it
    was started as a single process with --gpus n > 1; returns the launcher's
    exit status.  Rank 0 prints the JSON line."""
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def hbm_peak():
    """(GB/s, source): the measured copy bandwidth of MEASURED_PEAKS.json when
    the file is there, else the profiling recipe's fallback figure."""
    try:
        return float(json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, "fallback 6650 GB/s (no measured-peaks file on this machine)"


def workload_metric(wl) -> str:
    """The metric line of a workload (the N=2^16 key switch carries the
    headline metric's exact wording)."""
    if wl.name == "ntt_n16":
        return "forward+inverse negacyclic NTT throughput at N=2^16 (1 B200)"
    if wl.name == "sweep_n17":
        return "key-switches/s at N=2^17 level sweep 40..1 (1 B200)"
    if wl.op in ("rotate", "hoisted"):
        return (f"rotations/s at N=2^{wl.logN} ({'single' if wl.op == 'rotate' else f'{wl.n_rot} hoisted'}"
                " rotation(s) per ciphertext; 1 B200)")
    if wl.op == "bsgs":
        n1, n2 = wl.bsgs
        return (f"baby-step giant-step linear transforms/s at N=2^{wl.logN}, levels {wl.levels[0]}..{wl.levels[-1]} "
                f"({n2}x{n1} diagonals: {n1 - 1} hoisted baby and {n2 - 1} giant rotations each; 1 B200)")
    if wl.op == "relin":
        return f"ciphertext products (tensor + relinearisation) per second at N=2^{wl.logN} (1 B200)"
    if wl.logN == 16:
        return "key-switches/s at N=2^16 (1 B200); achieved HBM GB/s and % of roofline"
    return f"key-switches/s at N=2^{wl.logN} (1 B200)"


# --------------------------------------------------------------- our arm

def run_ours(args):
    import numpy as np
    import torch
    import datetime

    from key_switching_b200 import pc, synth

    world, rank, local = dist_setup()
    assert world == args.gpus, f"--gpus {args.gpus} but WORLD_SIZE={world}"
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    wl = synth.WORKLOADS[args.workload]
    plan = rank_plan(args.workload, wl.n_ct, world, rank, local)
    q, p = pc.chain(wl.logN, wl.bits, wl.L, wl.alpha)
    ctx = pc.Context(wl.logN, q, p, device=plan["device"])
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

    graphs = None
    items = list(plan["items"])
    if args.workload == "ntt_n16":
        unit, metric = "limb-NTTs/s", workload_metric(wl)
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
        run_op = None
    else:
        unit, metric = _unit(wl), workload_metric(wl)
        levels = list(wl.levels) if wl.levels else [L]
        B = len(items)  # this rank's ciphertexts per step
        nk = wl.n_rot if wl.op == "hoisted" else B  # keys per step
        if wl.op == "bsgs":
            nk = wl.bsgs[0] + wl.bsgs[1] - 2
            ctx.ensure_linear_transform_workspace(max(levels), wl.bsgs[0])
        else:
            ctx.ensure_workspace(max(levels), max(B, min(wl.n_rot, 16)) if wl.op == "hoisted" else B)
        per_set = (B * (2 * L * N * 4) * (2 if wl.op == "relin" else 1)
                   + nk * wl.dnum * (L + A) * N * 4 * (1 if regen else 2))
        nsets = max(2, math.ceil(2 * L2_BYTES / per_set)) if args.workload != "sweep_n17" else 1
        sets = []
        nct = B * (2 if wl.op == "relin" else 1)
        for s in range(nsets):
            key_ids = items if wl.op not in ("hoisted", "bsgs") else range(nk)
            keys = [make_key(1000 * s + k + 1) for k in key_ids]
            ct = dev(np.stack([np.stack([synth.uniform_residues(q, N, 50 + s, rank, k, h) for h in range(2)])
                               for k in (items if wl.op != "relin" else range(nct))]))
            sets.append((ct, keys))
        out = torch.empty((max(B, wl.n_rot), 2, L, N), dtype=torch.int32, device="cuda")
        units_per_step = (wl.n_rot if wl.op == "hoisted" else B) * len(levels)
        rot_gs = [pow(5, 1 << r, 2 * N) for r in range(wl.n_rot)]  # steps 1, 2, 4, ...
        diags = {}
        if wl.op == "bsgs":
            # per level: [n2][n1][l][N] uniform plaintext diagonals, drawn on
            # the device from a seeded generator (residue r of limb i mod q_i)
            n1, n2 = wl.bsgs
            gen = torch.Generator(device="cuda")
            gen.manual_seed(1234 + rank)
            qv = torch.tensor(q, dtype=torch.int64, device="cuda")
            for l in levels:
                r = torch.randint(0, 2**62, (n2, n1, l, N), generator=gen, device="cuda", dtype=torch.int64)
                diags[l] = (r % qv[:l].view(1, 1, l, 1)).to(torch.int32).contiguous()
            lt_gb = [pow(5, j, 2 * N) for j in range(1, n1)]           # baby rotations by 1 .. n1-1
            lt_gg = [pow(5, n1 * i, 2 * N) for i in range(1, n2)]      # giant rotations by n1, 2 n1, ...
            out_flat = out.view(-1)

        def run_op(ct, keys, st):
            """One step's library calls on stream st."""
            for l in levels:
                if wl.op == "rotate":
                    ctx.rotate(ct[0, 0, :l], ct[0, 1, :l], l, rot_gs[0], keys[0], out[0, 0, :l], out[0, 1, :l], st)
                elif wl.op == "hoisted":
                    ctx.rotate_hoisted(ct[0, 0, :l], ct[0, 1, :l], l, rot_gs, keys, out[:, :, :l], st)
                elif wl.op == "relin":
                    ctx.relinearize(ct[0, :, :l], ct[1, :, :l], l, keys[0], out[0, :, :l], st)
                elif wl.op == "bsgs":
                    n1 = wl.bsgs[0]
                    ctx.linear_transform(ct[0, 0, :l], ct[0, 1, :l], l, diags[l], lt_gb, keys[:n1 - 1], lt_gg,
                                         keys[n1 - 1:], out_flat[:2 * l * N].view(2, l, N), st)
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
            if graphs is not None:
                graphs[k % nsets].launch(stream)
            else:
                run_op(*sets[k % nsets], stream)
        # 6 launches per key switch (the inner product splits in two when the
        # ModDown branch overlaps), 5 when the stages run serially
        launches_per_step = (5 if os.environ.get("PC_NO_OVERLAP") else 6) * len(levels)
        if wl.op == "hoisted":  # one ModUp (2), then per batch of up to 16 rotations 4 (3 when serial)
            launches_per_step = (2 + (3 if os.environ.get("PC_NO_OVERLAP") else 4) * -(-wl.n_rot // 16)) \
                * len(levels)
        if wl.op == "bsgs":  # baby steps as hoisted rotations, one product kernel, a rotation per giant step
            n1, n2 = wl.bsgs
            fin = 3 if os.environ.get("PC_NO_OVERLAP") else 4
            launches_per_step = ((2 + fin * -(-(n1 - 1) // 16) if n1 > 1 else 0) + 1
                                 + (n2 - 1) * (2 + fin)) * len(levels)
        work = [op_counts(wl, l, regen) for l in levels]

    clocks = ClockSampler(local)
    clocks.start()
    # warm-up, then exactly K timed steps between barriers
    for k in range(args.warmup):
        step(k)
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
    ms = e0.elapsed_time(e1)
    ms = max_over_ranks(ms, dist, "cuda")
    value = whole_job_rate(units_per_step, args.steps, world, ms)
    if plan["scaling"] == "strong":
        # the ranks split one job's units: the job's units over the slowest rank's time
        value = wl.n_ct * len(levels) * args.steps / (ms * 1e-3)

    # per-kernel events: a separate pass of direct, instrumented calls after
    # the timed region (each runs its kernels serially on the stream, with an
    # event between consecutive kernels)
    stage_calls = []
    if run_op is not None and wl.op not in ("hoisted", "bsgs"):
        n_prof = max(10, min(args.steps, 30)) if len(levels) == 1 else 10
        for k in range(n_prof):
            ctx.profile_begin(len(levels), 1)
            run_op(*sets[k % nsets], stream)
            ms_k, n_k = ctx.profile_end()
            if n_k:
                stage_calls.append(ms_k)
    clk = clocks.stop()

    res = {"metric": metric, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
           "scaling": plan["scaling"], "vs_baseline": None, "dtype": "u32",
           "data": "synthetic (seeded uniform residues, uniform key 'b' halves; ChaCha12 seeds)",
           "config": {"workload": f"{wl.name}: N=2^{wl.logN}, L={L}, alpha={A}, dnum={wl.dnum}, "
                      f"{wl.n_ct} ct/step, levels {levels[0]}..{levels[-1]}, key a-half "
                      f"{'regenerated in-kernel (ChaCha12)' if regen else 'stored in HBM'}",
                      "l2": f"inputs rotated over {nsets} sets of {per_set / 1e6:.1f} MB (> 126 MB L2)",
                      "parallelism": (f"{wl.n_ct} (ciphertext, key) pairs split over {world} rank(s)"
                                      if plan["scaling"] == "strong" else f"replicas x{world}"),
                      "launch": "CUDA graph replay of every step" if graphs is not None else "library calls"},
           "gpu_launches": launches_per_step * args.steps, "clocks": clk}

    if args.workload == "ntt_n16":
        # forward + inverse NTT of 64 x 28 limbs: N/2 log N butterflies (one
        # modular multiply each) per limb and direction, plus the inverse's
        # N^-1 scale; bytes: every word read and written once per direction
        NPL = L + A
        mm = 2 * wl.n_ct * NPL * (N // 2 * wl.logN) + wl.n_ct * NPL * N
        by = 2 * 2 * wl.n_ct * NPL * N * 4
        sec_per_step = ms * 1e-3 / args.steps
        peak_derived = SMS * IMAD_PER_SM_CLK * 1965e6 / MODMUL_IMAD
        hbm, hbm_src = hbm_peak()
        t_roof = max(by / (hbm * 1e9), mm / peak_derived)
        res["step_roofline"] = {"modmuls_per_step": mm, "hbm_bytes_per_step": by,
                                "achieved_gbs": by / sec_per_step / 1e9,
                                "achieved_tmodmul_s": mm / sec_per_step / 1e12,
                                "t_roofline_us": t_roof * 1e6, "t_step_us": sec_per_step * 1e6,
                                "frac": t_roof / sec_per_step, "modmul_peak_derived": peak_derived,
                                "hbm_peak_gbs": hbm, "hbm_peak_source": hbm_src}
        peak_ops = SMS * ISSUE_LANES_PER_SM_CLK * 1965e6
        res["roofline"] = {"bound": "alu", "kernel": "whole step (column and row passes)",
                           "achieved": MODMUL_IMAD * mm / sec_per_step / 1e12, "peak": peak_ops / 1e12,
                           "unit": "Tintop/s", "frac": MODMUL_IMAD * mm / sec_per_step / peak_ops, "traffic": None,
                           "peak_source": "derived: 148 SMs x 128 issued 32-bit lane ops/clk x 1965 MHz; "
                                          "ops = 4 per Shoup modular multiply"}

    if work is not None:
        nct = B  # this rank's ciphertexts per step
        mm = sum(w["modmuls"] for w in work)
        by = sum(w["bytes"] for w in work)
        sec_per_step = ms * 1e-3 / args.steps
        peak_derived = SMS * IMAD_PER_SM_CLK * 1965e6 / MODMUL_IMAD
        try:
            peak_meas = pc.microbench(0, 2048, local) if rank == 0 else None
        except Exception:
            peak_meas = None
        hbm, hbm_src = hbm_peak()
        t_roof = max(by / (hbm * 1e9), mm / peak_derived)
        res["step_roofline"] = {"modmuls_per_step": mm * nct, "hbm_bytes_per_step": by * nct,
                                "achieved_gbs": by * nct / sec_per_step / 1e9,
                                "achieved_tmodmul_s": mm * nct / sec_per_step / 1e12,
                                "t_roofline_us": t_roof * nct * 1e6, "t_step_us": sec_per_step * 1e6,
                                "frac": t_roof * nct / sec_per_step,
                                "modmul_peak_derived": peak_derived,
                                "modmul_peak_microbench": peak_meas, "hbm_peak_gbs": hbm, "hbm_peak_source": hbm_src}
        peak_ops = SMS * ISSUE_LANES_PER_SM_CLK * 1965e6
        if stage_calls:
            smm = {}
            for l in levels:
                for kname, v in stage_modmuls(wl.logN, L, A, l).items():
                    smm[kname] = smm.get(kname, 0) + v * nct
            # integer lane operations per stage: 4 per modular multiply, 592
            # per ChaCha12 block (the inner-product stage regenerates a)
            blocks = sum(w["chacha_blocks"] for w in work) * nct
            sops = {k: MODMUL_IMAD * v for k, v in smm.items()}
            sops["inner_chacha"] += CHACHA_OPS * blocks
            med = {k: statistics.median(c[k] for c in stage_calls) for k in stage_calls[0]}
            tot = sum(med.values())
            top = max(med, key=med.get)
            per_launch_s = med[top] * 1e-3 / len(levels)
            ach = sops[top] / len(levels) / per_launch_s
            tr = KERNEL_TRAFFIC.get((args.workload, top)) if regen else None
            src_hash = kernel_source_hash()
            traffic = tr[0] if tr and tr[1] == src_hash else None
            res["roofline"] = {"bound": "alu", "kernel": top, "achieved": ach / 1e12,
                               "peak": peak_ops / 1e12, "unit": "Tintop/s",
                               "frac": ach / peak_ops,
                               "traffic": traffic,
                               "traffic_source": (f"ncu capture of the kernel sources hashing to {tr[1]} "
                                                  "(recorded constant, not measured in this run)"
                                                  if traffic is not None else
                                                  f"none recorded for kernel sources {src_hash}"),
                               "share": med[top] / tot if tot else None,
                               "ops_per_launch": sops[top] / len(levels),
                               "modmul_frac": smm[top] / len(levels) / per_launch_s / peak_derived,
                               "peak_source": "derived: 148 SMs x 128 issued 32-bit lane ops/clk (4 partitions x "
                                              "32; ALU + multiply-add pipes) x 1965 MHz; ops = 4 per Shoup "
                                              "modular multiply + 592 per ChaCha12 block"}
            res["stage_ms_per_step"] = med
            res["stage_sum_ms"] = tot
            res["stage_sampling"] = (f"median of {len(stage_calls)} direct instrumented steps run after the timed "
                                     "region (stages serial, one event between consecutive kernels)")
        else:
            # no per-kernel events on this path (hoisted rotations): the whole step
            ops = (MODMUL_IMAD * mm + CHACHA_OPS * sum(w["chacha_blocks"] for w in work)) * nct
            ach = ops / sec_per_step
            res["roofline"] = {"bound": "alu", "kernel": "whole step", "achieved": ach / 1e12,
                               "peak": peak_ops / 1e12, "unit": "Tintop/s", "frac": ach / peak_ops,
                               "traffic": None,
                               "peak_source": "derived: 148 SMs x 128 issued 32-bit lane ops/clk x 1965 MHz; "
                                              "ops = 4 per Shoup modular multiply + 592 per ChaCha12 block"}

    # end-to-end: host buffers through the library's host-buffer call, every
    # step's copies inside the timed region (pipelined with the key switches);
    # one call of 64 key switches, so that the first input copy and the last
    # output copy, which overlap nothing, weigh 1/64 of the call
    if not args.no_e2e and args.workload in ("rot1_n16", "relin_n12"):
        ct0, keys0 = sets[0]
        l = L
        ke = 64
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

    for g in graphs or []:
        g.close()
    if dist:
        dist.barrier()
        dist.destroy_process_group()

    # the oracle's CPU baseline: rank 0 of a single-GPU run only
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.workload in CPU_BASELINE_WORKLOADS:
        res["cpu_baseline"] = cpu_baseline(args.workload, budget_s=args.cpu_budget)
    if rank == 0:
        print(json.dumps(res), flush=True)


# ------------------------------------------------------------ oracle timing
# Everything below runs the CPU oracle only; it builds its own basis with the
# oracle's prime generator and imports nothing of the CUDA library.

CPU_BASELINE_WORKLOADS = ("rot1_n16", "relin_n12", "ntt_n16", "rotate_n16", "relin_mul_n12", "relin_mul_n16",
                          "hoisted8_n16", "batch16_n16", "sweep_n17", "bsgs_n17")


def _unit(wl):
    if wl.name == "ntt_n16":
        return "limb-NTTs/s"
    return {"rotate": "rotations/s", "hoisted": "rotations/s", "relin": "relinearisations/s",
            "bsgs": "linear-transforms/s"}.get(wl.op, "key-switches/s")


class OracleJob:
    """One operation of a workload on the oracle, with its seeded inputs: a key
    switch (rotation, relinearisation, hoisted rotations) at the workload's
    top level, or for the NTT workload a forward + inverse NTT of one limb."""

    def __init__(self, name: str, tag: int = 0):
        import numpy as np
        from key_switching_b200 import synth
        from oracle import oracle as O
        self.O, self.np = O, np
        wl = synth.WORKLOADS[name]
        self.wl = wl
        P = O.chain(wl.logN, wl.bits, wl.L, wl.alpha)
        self.P = P
        prim = [P.prime(g) for g in range(P.L + P.alpha)]
        self.l = wl.L
        if name == "ntt_n16":
            self.x = synth.uniform_residues(prim[:1], P.N, 40, tag)[0]
            self.q = prim[0]
            return
        self.b = np.stack([synth.uniform_residues(prim, P.N, 1, 0xB, j) for j in range(P.dnum)])
        if wl.op == "bsgs":
            # a bounded sample of the level sweep: transforms at its mean level
            self.l = sum(wl.levels) // len(wl.levels)
            n1, n2 = wl.bsgs
            self.diag = np.stack([np.stack([synth.uniform_residues(P.q[:self.l], P.N, 52, tag, i, j)
                                            for j in range(n1)]) for i in range(n2)])
        self.c0 = synth.uniform_residues(P.q[:self.l], P.N, 50, tag, 0, 0)
        self.c1 = synth.uniform_residues(P.q[:self.l], P.N, 50, tag, 0, 1)
        self.y0 = synth.uniform_residues(P.q[:self.l], P.N, 51, tag, 0, 0)
        self.y1 = synth.uniform_residues(P.q[:self.l], P.N, 51, tag, 0, 1)
        self.seed = synth.chacha_seed(1, tag)

    def run(self) -> int:
        """Run one operation; returns the number of units done."""
        O, P, wl, l = self.O, self.P, self.wl, self.l
        if wl.name == "ntt_n16":
            y = O.ntt_fwd(self.x, P.logN, self.q)
            O.ntt_inv(y, P.logN, self.q)
            return 2
        if wl.op == "rotate":
            O.rotate(P, self.c0, self.c1, l, pow(5, 1, 2 * P.N), self.seed, self.b)
        elif wl.op == "hoisted":
            gs = [pow(5, 1 << r, 2 * P.N) for r in range(wl.n_rot)]
            O.rotate_hoisted(P, self.c0, self.c1, l, gs, [self.seed] * wl.n_rot, [self.b] * wl.n_rot)
            return wl.n_rot
        elif wl.op == "relin":
            O.relinearize(P, self.c0, self.c1, self.y0, self.y1, l, self.seed, self.b)
        elif wl.op == "bsgs":
            n1, n2 = wl.bsgs
            gb = [pow(5, j, 2 * P.N) for j in range(1, n1)]
            gg = [pow(5, n1 * i, 2 * P.N) for i in range(1, n2)]
            O.linear_transform(P, self.c0, self.c1, l, self.diag, gb, [self.seed] * (n1 - 1), [self.b] * (n1 - 1),
                               gg, [self.seed] * (n2 - 1), [self.b] * (n2 - 1))
        else:
            O.keyswitch(P, self.c0, self.c1, l, self.seed, self.b)
        return 1


def _oracle_worker(name, tag, budget_s, start, q):
    """A worker process: set up, wait for the others, run whole operations for
    about budget_s seconds (at least one), report (units, seconds)."""
    try:
        job = OracleJob(name, tag)
        start.wait()
        t0 = time.perf_counter()
        n = 0
        while True:
            n += job.run()
            dt = time.perf_counter() - t0
            if dt >= budget_s:
                break
        q.put((n, dt))
    except BaseException as e:  # report, do not hang the parent
        q.put((0, repr(e)))


def oracle_rate(name: str, workers: int, budget_s: float):
    """Units per second of the oracle on `workers` host processes running
    independent operations at once: (units summed over the workers) / (the
    slowest worker's time).  Single-threaded when workers == 1 (in process)."""
    if workers == 1:
        job = OracleJob(name)
        t0 = time.perf_counter()
        n = 0
        while True:
            n += job.run()
            dt = time.perf_counter() - t0
            if dt >= budget_s:
                break
        return n / dt, n, dt
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    start = ctx.Barrier(workers)
    q = ctx.Queue()
    procs = [ctx.Process(target=_oracle_worker, args=(name, w, budget_s, start, q)) for w in range(workers)]
    for p in procs:
        p.start()
    res = [q.get(timeout=600 + 4 * budget_s) for _ in procs]
    for p in procs:
        p.join(timeout=60)
    bad = [r for r in res if not isinstance(r[1], float)]
    if bad:
        raise RuntimeError(f"oracle worker failed: {bad[0][1]}")
    n = sum(r[0] for r in res)
    dt = max(r[1] for r in res)
    return n / dt, n, dt


def host_cpu():
    """(logical cores, CPU model) of this host."""
    model = "unknown"
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                model = ln.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return os.cpu_count() or 1, model


def cpu_baseline(name: str, budget_s: float = 10.0):
    """The oracle as it stands on this host's cores, on bounded samples of the
    workload: single-threaded, and one independent operation per core on all
    cores (the headline value); also the two other small workloads named by
    the survey (N=2^12 key switch, N=2^16 NTT) with the same method."""
    cores, model = host_cpu()
    workers = min(cores, 64)
    from key_switching_b200 import synth
    wl = synth.WORKLOADS[name]
    unit = _unit(wl)
    v1, n1, t1 = oracle_rate(name, 1, budget_s)
    va, na, ta = oracle_rate(name, workers, budget_s)
    out = {"value": va, "unit": unit, "cores": workers, "kind": "oracle", "cpu_model": model, "nproc": cores,
           "sample": f"{na} operation(s) of {name} (top level) on {workers} processes in {ta:.1f} s; "
                     f"single thread: {n1} in {t1:.1f} s",
           "single_thread": {"value": v1, "unit": unit, "cores": 1}}
    others = {}
    for other in ("relin_n12", "ntt_n16"):
        if other == name:
            continue
        ow = synth.WORKLOADS[other]
        s1 = oracle_rate(other, 1, budget_s / 4)
        sa = oracle_rate(other, workers, budget_s / 4)
        others[other] = {"unit": _unit(ow), "single_thread": s1[0], "all_cores": sa[0], "cores": workers,
                         "sample": f"{s1[1]} unit(s) in {s1[2]:.1f} s on 1 thread; {sa[1]} in {sa[2]:.1f} s "
                                   f"on {workers} processes"}
    out["other_workloads"] = others
    return out


def run_reference(args):
    """The oracle on the host cores, on this arm's workload, metric and unit:
    one independent operation per core at a time, each step a bounded sample."""
    world, rank, local = dist_setup()
    if rank != 0:
        return
    from key_switching_b200 import synth
    wl = synth.WORKLOADS[args.workload]
    cores, model = host_cpu()
    workers = min(cores, 64)
    unit = _unit(wl)
    # a few seconds per step, the whole run within a few minutes
    budget = max(2.0, min(12.0, 150.0 / max(1, args.steps)))
    v, n, dt = oracle_rate(args.workload, workers, budget * max(1, args.steps))
    metric = workload_metric(wl)
    sample = (f"{n} unit(s) of {wl.name} (top level) on {workers} processes, one independent operation per "
              f"process at a time, in {dt:.1f} s ({args.steps} step(s) of ~{budget:.0f} s requested)")
    res = {"impl": "reference", "metric": metric,
           "value": v, "unit": unit, "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": dt * 1e3 / max(1, args.steps), "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "u32", "data": "synthetic",
           "config": {"workload": f"{wl.name}: N=2^{wl.logN}, L={wl.L}, alpha={wl.alpha}, dnum={wl.dnum}, "
                      "operations at the top level, key a-half regenerated (ChaCha12)"},
           "cpu_baseline": {"value": v, "unit": unit, "cores": workers, "kind": "oracle", "cpu_model": model,
                            "nproc": cores, "sample": sample},
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
                             "hoisted8_n16", "relin_mul_n12", "relin_mul_n16", "bsgs_n17"])
    ap.add_argument("--keys", default="regen", choices=["regen", "stored"])
    ap.add_argument("--no-graph", action="store_true",
                    help="call the library every step instead of replaying a CUDA graph of the step")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=8.0, help="seconds of oracle work per cpu_baseline sample")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
        return
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(launch_ranks(sys.argv[1:], args.gpus))
    run_ours(args)


if __name__ == "__main__":
    main()
