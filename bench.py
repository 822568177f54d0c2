"""Benchmark: RNS-CKKS hybrid key switching at N=2^16, full level, on B200.

One step = one pass of the whole key-switching path over one batch of B independent units
of the N=2^16 full-level workload (`n16-full`; default B = 8), each unit
  d   = tensor(x, y)            (ct x ct product, 36 limbs)
  r   = relin(d)                (key switch #1: ModUp, ChaCha12 inner product, ModDown)
  out = rotate(r, g = 5)        (automorphism + key switch #2)
at N=2^16, 36 ciphertext + 12 special primes (< 2^30), dnum 3, full level.  The batch runs
through the batched entry points (one launch per kernel covers all B units).  Every unit has
its own relinearisation and rotation keys.  The metric is key-switches/s (2 per unit) over all
ranks; rotations/s is reported beside it.

Inputs are synthetic: uniform residues for the ciphertexts and for the keys' stored b halves
(the cost of every kernel is data independent), seeded per rank.  Three independent buffer
and key sets (each larger than the 126 MB L2) are cycled so that consecutive steps never find
their inputs in L2.

--impl reference times the CPU oracle (the plain C restatement of the same path) on the host
cores instead, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

CONFIG_KEY = "n16-full"
METRIC = "key-switches/s (rotations/s) at N=2^16, 32-bit RNS; % of HBM roofline"
KS_PER_UNIT = 2          # relin + rotation
ROT_PER_UNIT = 1
N_SETS = 3


def _env_int(name, default):
    try:
        return int(os.environ.get(name, default))
    except ValueError:
        return default


def rank_env():
    """(rank, world, local_rank) from the torchrun environment (1 process when absent)."""
    return _env_int("RANK", 0), _env_int("WORLD_SIZE", 1), _env_int("LOCAL_RANK", 0)


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (the job's time is its slowest rank's)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: int, world: int, ms_max: float) -> float:
    """Whole-job throughput: every rank processes its own units (weak scaling, replicas); the
    job takes the slowest rank's time."""
    return units_per_rank * world / (ms_max / 1e3)


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import fhe_key_switching_b200 as ks

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    cfg = W.CONFIGS[CONFIG_KEY]
    n, lvl = cfg.n, cfg.level
    na = lvl + 1
    q, p = ks.ckks_gen_primes(cfg.log_n, cfg.n_q, cfg.n_p)
    ctx = ks.Context(cfg.log_n, q, p, cfg.dnum)
    g = ks.galois_element(cfg.log_n, cfg.rot_steps[0])
    nd = -(-cfg.n_q // cfg.alpha)
    mods = q + p

    def residues(moduli, seed_tag):
        a = W.uniform_residues(moduli, n, W.rng(cfg.seed, W.TAG_SYNTH, rank, seed_tag))
        return torch.from_numpy(a).to(dev)

    B = args.batch
    sets = []
    for s in range(N_SETS):
        x = residues(q[:na] * 2 * B, 10 * s + 1).view(B, 2, na, n)
        y = residues(q[:na] * 2 * B, 10 * s + 2).view(B, 2, na, n)
        b_rel = residues(mods * nd * B, 10 * s + 3).view(B, nd, len(mods), n)
        b_rot = residues(mods * nd * B, 10 * s + 4).view(B, nd, len(mods), n)
        # --stored-a (ablation): the keys carry a stored a half read from HBM instead of ChaCha12
        a_rel = residues(mods * nd * B, 10 * s + 5).view(B, nd, len(mods), n) if args.stored_a else None
        a_rot = residues(mods * nd * B, 10 * s + 6).view(B, nd, len(mods), n) if args.stored_a else None
        # every unit has its own key pair: its own seed (so its own regenerated a half) and b half
        seeds = [hashlib.sha256(cfg.chacha_seed + bytes([s, i])).digest() for i in range(B)]
        sets.append(dict(x=x, y=y, b_rel=b_rel, b_rot=b_rot, a_rel=a_rel, a_rot=a_rot,
                         k_rel=[ks.make_evk(b_rel[i], seeds[i], 0,
                                            a=a_rel[i] if args.stored_a else None) for i in range(B)],
                         k_rot=[ks.make_evk(b_rot[i], seeds[i], g,
                                            a=a_rot[i] if args.stored_a else None) for i in range(B)]))
    d = torch.empty((B, 3, na, n), dtype=torch.uint32, device=dev)
    r = torch.empty((B, 2, na, n), dtype=torch.uint32, device=dev)
    out = torch.empty((B, 2, na, n), dtype=torch.uint32, device=dev)
    # the batch runs as S sub-batches of B/S units, one per CUDA stream, so that one sub-batch's
    # ALU-bound kernels overlap another's memory-bound ones
    S = args.streams if args.streams is not None else (2 if B % 2 == 0 else 1)
    if S < 1 or B % S:
        raise SystemExit(f"--streams {S} must divide --batch {B}")
    Bs = B // S
    main = torch.cuda.current_stream(dev)
    streams = [main] + [torch.cuda.Stream(dev) for _ in range(S - 1)]
    wss = [ctx.workspace(lvl, Bs, device=dev) for _ in range(S)]
    gal = [g] * Bs

    def sub(si):
        return slice(si * Bs, (si + 1) * Bs)

    def step_on(si, st, x, y, stream):
        z = sub(si)
        ks.ckks_tensor_batch(ctx, Bs, x[z], y[z], lvl, d[z], stream)
        ks.ckks_relin_batch(ctx, d[z], lvl, st["k_rel"][z], r[z], wss[si], stream)
        ks.ckks_rotate_batch(ctx, r[z], lvl, gal, st["k_rot"][z], out[z], wss[si], stream)

    def step(i, n_streams=S):
        st = sets[i % N_SETS]
        if n_streams == 1:          # the same work, every sub-batch on the main stream in turn
            for si in range(S):
                step_on(si, st, st["x"], st["y"], main)
            return
        for si in range(S):
            step_on(si, st, st["x"], st["y"], streams[si])

    def fork():
        ev = torch.cuda.Event()
        ev.record(main)
        for s_ in streams[1:]:
            s_.wait_event(ev)

    def join():
        for s_ in streams[1:]:
            ev = torch.cuda.Event()
            ev.record(s_)
            main.wait_event(ev)

    def barrier():
        if world > 1:
            dist.barrier()

    def timed(fn, steps):
        """Device time of `steps` calls of fn (ms, max over ranks), events on the main stream."""
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(main)
        fork()
        for i in range(steps):
            fn(i)
        join()
        e1.record(main)
        torch.cuda.synchronize()
        barrier()
        return max_over_ranks(e0.elapsed_time(e1), world, dev)

    fork()
    for i in range(args.warmup):
        step(i)
    join()
    torch.cuda.synchronize()
    barrier()
    # with --graph the timed steps replay one CUDA graph per input set: the whole multi-stream
    # step (fork, every sub-batch's launches on its stream, join) captured once
    graphs = []
    if args.graph:
        cap = torch.cuda.Stream(dev)
        for si_set in range(N_SETS):
            gph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gph, stream=cap):
                ev = torch.cuda.Event()
                ev.record(cap)
                for s_ in streams[1:]:
                    s_.wait_event(ev)
                st = sets[si_set]
                for si in range(S):
                    step_on(si, st, st["x"], st["y"], cap if si == 0 else streams[si])
                for s_ in streams[1:]:
                    ev = torch.cuda.Event()
                    ev.record(s_)
                    cap.wait_event(ev)
            graphs.append(gph)
        torch.cuda.synchronize()

    def step_timed(i):
        if graphs:
            graphs[i % N_SETS].replay()
        else:
            step(i)

    for i in range(args.warmup):
        step_timed(i)
    torch.cuda.synchronize()
    barrier()
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    # the dominant kernel's launches inside the timed region (overlapped with the other streams);
    # graph replays carry no profiling events, so this figure exists for eager steps only
    ks.ckks_prof_begin(ctx, DOMINANT, KS_PER_UNIT * S * args.steps)
    ms = timed(step_timed, args.steps)
    dom_launches_ov, dom_ms_ov = ks.ckks_prof_end(ctx)
    # the dominant kernel alone: the same steps with every launch on the main stream, so that
    # each launch's events bracket that kernel only
    ks.ckks_prof_begin(ctx, DOMINANT, KS_PER_UNIT * S * args.steps)
    ms_single = timed(lambda i: step(i, 1), args.steps)
    dom_launches, dom_ms = ks.ckks_prof_end(ctx)
    clk = clocks.stop()
    ms_per_step = ms / args.steps
    value = job_throughput(KS_PER_UNIT * B * args.steps, world, ms)

    # end to end: pinned host inputs copied in, result copied out, every step; each stream
    # copies its own sub-batch
    h_x = [s["x"].cpu().pin_memory() for s in sets]
    h_y = [s["y"].cpu().pin_memory() for s in sets]
    h_out = torch.empty((B, 2, na, n), dtype=torch.uint32).pin_memory()
    dx, dy = torch.empty_like(sets[0]["x"]), torch.empty_like(sets[0]["y"])

    def step_e2e(i):
        st = sets[i % N_SETS]
        for si in range(S):
            z = sub(si)
            with torch.cuda.stream(streams[si]):
                dx[z].copy_(h_x[i % N_SETS][z], non_blocking=True)
                dy[z].copy_(h_y[i % N_SETS][z], non_blocking=True)
            step_on(si, st, dx, dy, streams[si])
            with torch.cuda.stream(streams[si]):
                h_out[z].copy_(out[z], non_blocking=True)

    fork()
    for i in range(args.warmup):
        step_e2e(i)
    join()
    ms_e2e = timed(step_e2e, args.steps)
    e2e_value = job_throughput(KS_PER_UNIT * B * args.steps, world, ms_e2e)
    h2d = (sets[0]["x"].numel() + sets[0]["y"].numel()) * 4
    d2h = out.numel() * 4

    cpu = cpu_baseline() if (rank == 0 and world == 1 and not args.no_cpu_baseline) else None

    if rank == 0:
        line = {
            "metric": METRIC,
            "value": value,
            "unit": "key-switches/s",
            "rotations_per_s": job_throughput(ROT_PER_UNIT * B * args.steps, world, ms),
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms_per_step,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "u32",
            "data": "synthetic",
            "config": dict(workload_config(cfg, B, world, args.stored_a, f"{S} CUDA streams x {Bs} units"),
                           launch="one CUDA graph replay per step (captured per input set)" if graphs
                           else "eager launches"),
            "e2e": {"value": e2e_value, "unit": "key-switches/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": args.steps * LAUNCHES_PER_STEP * S,
            "kernel_launches_note": "one launch per kernel covers the whole batch",
            "clocks": clk,
            "roofline": roofline(cfg, dom_launches, dom_ms, clk, Bs, ms_single / args.steps,
                                 dom_launches_ov, dom_ms_ov),
            "hbm_fraction_step": {"b_min_bytes_per_step": B * step_bytes_min(cfg),
                                  "frac": B * step_bytes_min(cfg) / (ms_per_step / 1e3) / (HBM_PEAK_GBS * 1e9),
                                  "peak_gbs": HBM_PEAK_GBS, "peak_source": PEAK_SOURCE},
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


DOMINANT = "ip_row"      # the fused NTT-row-pass + ChaCha12 + key inner-product kernel


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d.get("sm_max_mhz", 1965.0)), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1965.0, "fallback"


HBM_PEAK_GBS, SM_MAX_MHZ, PEAK_SOURCE = _peaks()
N_SM = 148


def alu_peak_tops(mhz: float) -> float:
    """int32 issue peak: 148 SMs x 4 sub-partitions x 32 lanes x 1 instruction/clock."""
    return N_SM * 4 * 32 * mhz * 1e6 / 1e12


def ip_row_ops(cfg) -> float:
    """Algorithmic int32 operations of one key switch's share of a k_ip_row launch, with the unit costs
    of the op model: ChaCha12 block 608 (8 coefficients), 64-bit word reduction 8, NTT butterfly
    8, variable modular product 6, modular addition 2.  Units: beta*ext (digit, limb) pairs of N
    coefficients; the row pass (8 of log N stages) runs on the pairs outside their digit."""
    na = cfg.level + 1
    ext = na + cfg.n_p
    beta = -(-na // cfg.alpha)
    pairs = beta * ext
    n = cfg.n
    chacha = pairs * n / 8 * 608
    a_red = pairs * n * 8
    ntt = (pairs - na) * 8 * (n / 2) * 8
    macs = 2 * pairs * n * 6 + 2 * pairs * n * 2
    return chacha + a_red + ntt + macs


def roofline(cfg, launches, total_ms, clk, batch, single_step_ms, launches_ov, total_ms_ov):
    """The dominant kernel against the int32 ALU issue peak.  `launches`/`total_ms`: its launches
    in a single-stream pass of the timed steps (each launch's events bracket that kernel only);
    `launches_ov`/`total_ms_ov`: the same kernel inside the timed multi-stream region, where its
    events also span the other streams' concurrent kernels."""
    if not launches:
        return None
    avg_s = total_ms / launches / 1e3
    achieved = batch * ip_row_ops(cfg) / avg_s / 1e12
    peak = alu_peak_tops(SM_MAX_MHZ)
    out = {"kernel": "k_ip_row (ModUp last NTT pass + ChaCha12 + key inner product)",
           "bound": "alu", "achieved": achieved, "peak": peak, "unit": "Tops (int32)",
           "frac": achieved / peak,
           "traffic": None if IP_ROW_TRAFFIC_PER_UNIT is None else IP_ROW_TRAFFIC_PER_UNIT * batch,
           "units_per_launch": batch,
           "launches": launches,
           "avg_launch_us": avg_s * 1e6,
           "timed_in": "single-stream pass of the timed steps, right after the timed region "
                       f"({single_step_ms:.3f} ms per step)",
           "peak_source": f"derived: {N_SM} SMs x 128 int32 lanes x {SM_MAX_MHZ:.0f} MHz"}
    if launches_ov:
        out["in_timed_region"] = {"launches": launches_ov,
                                  "avg_launch_us": total_ms_ov / launches_ov * 1e3,
                                  "note": "overlapped with the other streams' kernels"}
    return out


# DRAM bytes (read + write) per unit of a k_ip_row launch, from an ncu launch list of this
# benchmark (4-unit launches; mean of 20: dram__bytes_read 392.51 MB + write 78.97 MB), scaled
# by the units a launch covers; None when the kernel changed after the capture.
IP_ROW_TRAFFIC_PER_UNIT = 471.48e6 / 4


def step_bytes_min(cfg) -> int:
    """Compulsory HBM bytes of one step: inputs, the keys' stored b halves and outputs of the
    tensor product (4 -> 3 polys), the relinearisation (3 polys + key -> 2) and the rotation
    (2 polys + key -> 2); the a halves are regenerated, intermediates are not counted."""
    na = cfg.level + 1
    nd = -(-cfg.n_q // cfg.alpha)
    key = nd * (cfg.n_q + cfg.n_p)
    limbs = (4 + 3) * na + (3 * na + key + 2 * na) + (2 * na + key + 2 * na)
    return limbs * cfg.n * 4


# kernels launched by one step: tensor (1) + 2 key switches x 10 (ModUp 4, inner product with
# the last ModUp and first ModDown NTT passes 2, ModDown 4 including the fused combine)
LAUNCHES_PER_STEP = 1 + 2 * 10


def run_workload(args, local_rank):
    """Informational throughput (not the benchmark's headline line):
    n16-bsgs32 = 32 hoisted rotations of one ciphertext at level 24 (one ModUp, 32 keys);
    n16-stream64 = 64 pairs, each tensor + relin + rotate by 2^(i mod 15), level 20, dnum 4
        (one relinearisation key, 15 rotation keys, all as batched calls);
    n16-stream64-rescale = the same with a rescale after the relinearisation (rotation at
        level 19);
    rescale = 64 rescales of level-35 ciphertexts on the N=2^16 full-level chain per step;
    bsgs = one baby-step giant-step transform with n16-bsgs32's 32 keys (baby steps 0..15,
        giant steps 16 j for j = 0..17: 288 plaintext diagonals over the extended basis,
        level 24);
    bsgs-n14 = the same transform shape on the N=2^14 chain (level 11), a smaller case whose
        plaintexts (302 MB) still exceed L2, for profiling."""
    import torch
    import fhe_key_switching_b200 as ks

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    key = str(args.workload)
    cfg = W.CONFIGS[{"n16-stream64-rescale": "n16-stream64", "rescale": "n16-full", "bsgs": "n16-bsgs32",
                     "bsgs-n14": "n14-hoisted8"}.get(key, key)]
    n, lvl = cfg.n, cfg.level
    na = lvl + 1
    q, p = ks.ckks_gen_primes(cfg.log_n, cfg.n_q, cfg.n_p)
    ctx = ks.Context(cfg.log_n, q, p, cfg.dnum)
    nd = -(-cfg.n_q // cfg.alpha)
    mods = q + p
    gen = W.rng(cfg.seed, W.TAG_SYNTH, 7)

    def res(moduli):
        return torch.from_numpy(W.uniform_residues(moduli, n, gen)).to(dev)

    steps_g = sorted(set(cfg.rot_steps), key=cfg.rot_steps.index)
    gal = {r: ks.galois_element(cfg.log_n, r) for r in steps_g}
    keys_t = {r: res(mods * nd).view(nd, len(mods), n) for r in steps_g}
    evk = {r: ks.make_evk(keys_t[r], cfg.chacha_seed, gal[r]) for r in steps_g}
    stream = torch.cuda.current_stream(dev)
    if key == "n16-bsgs32":
        cts = [res(q[:na] * 2).view(2, na, n) for _ in range(N_SETS)]
        R = len(cfg.rot_steps)
        gs = [gal[r] for r in cfg.rot_steps]
        ev = [evk[r] for r in cfg.rot_steps]
        out = torch.empty((R, 2, na, n), dtype=torch.uint32, device=dev)
        ws = ctx.workspace(lvl, R, device=dev)

        def step(i):
            ks.ckks_rotate_hoisted(ctx, cts[i % N_SETS], lvl, gs, ev, out, ws, stream)
        ks_per_step, rot_per_step = R, R
    elif key == "n16-stream64":
        P_ = cfg.n_pairs
        xs = [res(q[:na] * 2 * P_).view(P_, 2, na, n) for _ in range(2)]
        ys = [res(q[:na] * 2 * P_).view(P_, 2, na, n) for _ in range(2)]
        b_rel = res(mods * nd).view(nd, len(mods), n)
        k_rel = ks.make_evk(b_rel, cfg.chacha_seed, 0)
        d = torch.empty((P_, 3, na, n), dtype=torch.uint32, device=dev)
        r1 = torch.empty((P_, 2, na, n), dtype=torch.uint32, device=dev)
        out = torch.empty((P_, 2, na, n), dtype=torch.uint32, device=dev)
        ws = ctx.workspace(lvl, P_, device=dev)
        gs = [gal[r] for r in cfg.rot_steps]
        ev = [evk[r] for r in cfg.rot_steps]

        def step(i):
            ks.ckks_tensor_batch(ctx, P_, xs[i % 2], ys[i % 2], lvl, d, stream)
            ks.ckks_relin_batch(ctx, d, lvl, [k_rel] * P_, r1, ws, stream)
            ks.ckks_rotate_batch(ctx, r1, lvl, gs, ev, out, ws, stream)
        ks_per_step, rot_per_step = 2 * P_, P_
    elif key == "n16-stream64-rescale":
        P_ = cfg.n_pairs
        xs = [res(q[:na] * 2 * P_).view(P_, 2, na, n) for _ in range(2)]
        ys = [res(q[:na] * 2 * P_).view(P_, 2, na, n) for _ in range(2)]
        b_rel = res(mods * nd).view(nd, len(mods), n)
        k_rel = ks.make_evk(b_rel, cfg.chacha_seed, 0)
        d = torch.empty((P_, 3, na, n), dtype=torch.uint32, device=dev)
        r1 = torch.empty((P_, 2, na, n), dtype=torch.uint32, device=dev)
        r2 = torch.empty((P_, 2, lvl, n), dtype=torch.uint32, device=dev)
        out = torch.empty((P_, 2, lvl, n), dtype=torch.uint32, device=dev)
        ws = ctx.workspace(lvl, P_, device=dev)
        gs = [gal[r] for r in cfg.rot_steps]
        ev = [evk[r] for r in cfg.rot_steps]

        def step(i):
            ks.ckks_tensor_batch(ctx, P_, xs[i % 2], ys[i % 2], lvl, d, stream)
            ks.ckks_relin_batch(ctx, d, lvl, [k_rel] * P_, r1, ws, stream)
            ks.ckks_rescale_batch(ctx, P_, r1, lvl, r2, ws, stream)
            ks.ckks_rotate_batch(ctx, r2, lvl - 1, gs, ev, out, ws, stream)
        ks_per_step, rot_per_step = 2 * P_, P_
    elif key == "rescale":
        R = 64
        cts = [res(q[:na] * 2 * R).view(R, 2, na, n) for _ in range(N_SETS)]
        out = torch.empty((R, 2, lvl, n), dtype=torch.uint32, device=dev)
        ws = ctx.workspace(lvl, R, device=dev)

        def step(i):
            ks.ckks_rescale_batch(ctx, R, cts[i % N_SETS], lvl, out, ws, stream)
        ks_per_step, rot_per_step = 0, 0
    elif key in ("bsgs", "bsgs-n14"):
        n1, n2 = 16, 18
        baby = [1] + [ks.galois_element(cfg.log_n, k) for k in range(1, n1)]
        giant = [1] + [ks.galois_element(cfg.log_n, n1 * j) for j in range(1, n2)]
        gk = {g: ks.make_evk(res(mods * nd).view(nd, len(mods), n), cfg.chacha_seed, g)
              for g in baby + giant if g != 1}
        ext = na + cfg.n_p
        pt = res((q[:na] + p) * n2 * n1).view(n2, n1, ext, n)
        cts = [res(q[:na] * 2).view(2, na, n) for _ in range(N_SETS)]
        out = torch.empty((2, na, n), dtype=torch.uint32, device=dev)
        ws = ks.ckks_bsgs_workspace(ctx, lvl, n1, n2, device=dev)
        bk = [gk.get(g) for g in baby]
        gkk = [gk.get(g) for g in giant]

        def step(i):
            ks.ckks_bsgs(ctx, cts[i % N_SETS], lvl, baby, bk, giant, gkk, pt, out, ws, stream)
        ks_per_step, rot_per_step = (n1 - 1) + (n2 - 1), (n1 - 1) + (n2 - 1)
    else:
        raise SystemExit(f"--workload {key}: use n16-full (default), n16-bsgs32, n16-stream64, "
                         "n16-stream64-rescale, rescale, bsgs or bsgs-n14")
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if key in ("bsgs", "bsgs-n14"):
        ks.ckks_prof_begin(ctx, "bsgs_combine", args.steps)
    e0.record(stream)
    for i in range(args.steps):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    if key in ("bsgs", "bsgs-n14"):
        launches, comb_ms = ks.ckks_prof_end(ctx)
        # compulsory bytes of one combine launch: every plaintext once, the 15 rotated babies'
        # accumulators and the input ciphertext once, the 18 giant sums written once
        b_comb = (n2 * n1 * ext + (n1 - 1) * 2 * ext + 2 * na + n2 * 2 * ext) * n * 4
        comb_s = comb_ms / max(launches, 1) / 1e3
        print(json.dumps({"workload": f"bsgs: {cfg.key} chain, N=2^{cfg.log_n}, {n1} baby x {n2} giant "
                                      f"steps, level {lvl}",
                          "informational": True, "transforms_per_s": args.steps / (ms / 1e3),
                          "ms_per_step": ms / args.steps, "steps": args.steps, "warmup": args.warmup,
                          "rotations_per_transform": ks_per_step,
                          "combine_kernel": {"avg_launch_us": comb_s * 1e6, "launches": launches,
                                             "bytes_per_launch": b_comb, "achieved_gbs": b_comb / comb_s / 1e9,
                                             "peak_gbs": HBM_PEAK_GBS,
                                             "frac": b_comb / comb_s / 1e9 / HBM_PEAK_GBS,
                                             "share_of_step": comb_s * 1e3 / (ms / args.steps)},
                          "clocks": clk}), flush=True)
        return
    if key == "rescale":
        # compulsory bytes per rescale: read 2(l+1) limbs, write 2l limbs
        b_min = (2 * na + 2 * lvl) * n * 4
        per_s = R * args.steps / (ms / 1e3)
        print(json.dumps({"workload": f"rescale: N=2^{cfg.log_n}, level {lvl} -> {lvl - 1}, {R} per step",
                          "informational": True, "rescales_per_s": per_s, "ms_per_step": ms / args.steps,
                          "steps": args.steps, "warmup": args.warmup,
                          "hbm": {"b_min_bytes_per_rescale": b_min, "achieved_gbs": b_min * per_s / 1e9,
                                  "peak_gbs": HBM_PEAK_GBS, "frac": b_min * per_s / 1e9 / HBM_PEAK_GBS},
                          "clocks": clk}), flush=True)
        return
    print(json.dumps({"workload": key, "informational": True,
                      "key_switches_per_s": ks_per_step * args.steps / (ms / 1e3),
                      "rotations_per_s": rot_per_step * args.steps / (ms / 1e3),
                      "ms_per_step": ms / args.steps, "steps": args.steps, "warmup": args.warmup,
                      "key_switches_per_step": ks_per_step, "clocks": clk}), flush=True)


def _oracle_sample():
    """Bounded CPU sample of the same step: one relinearisation and one rotation of n16-full,
    timed on the oracle with synthetic residues (cost is data independent)."""
    import numpy as np
    import oracle

    cfg = W.CONFIGS[CONFIG_KEY]
    ctx = oracle.Ctx(cfg.log_n, cfg.n_q, cfg.n_p)
    n, lvl = cfg.n, cfg.level
    na = lvl + 1
    nd = -(-cfg.n_q // cfg.alpha)
    gen = W.rng(cfg.seed, W.TAG_SYNTH, 99)
    x = W.uniform_residues(ctx.q[:na] * 2, n, gen).reshape(2, na, n)
    y = W.uniform_residues(ctx.q[:na] * 2, n, gen).reshape(2, na, n)
    b = W.uniform_residues(ctx.mod * nd, n, gen).reshape(nd, len(ctx.mod), n)
    g = ctx.galois(1)

    def one_step():
        dd = ctx.tensor(x, y, lvl)
        rr = ctx.relin(dd, lvl, cfg.alpha, b, cfg.chacha_seed, 0)
        ctx.rotate(rr, lvl, cfg.alpha, g, b, cfg.chacha_seed, g)

    return one_step


def _omp_threads():
    v = os.environ.get("OMP_NUM_THREADS")
    return int(v) if v and v.isdigit() else (os.cpu_count() or 1)


def cpu_baseline(max_seconds: float = 20.0):
    one_step = _oracle_sample()
    one_step()                              # warm (tables, page faults)
    t0 = time.perf_counter()
    k = 0
    while True:
        one_step()
        k += 1
        if time.perf_counter() - t0 > max_seconds / 2 or k >= 8:
            break
    dt = time.perf_counter() - t0
    return {"value": KS_PER_UNIT * k / dt, "unit": "key-switches/s", "cores": _omp_threads(),
            "kind": "oracle",
            "sample": f"{k} units of the N=2^16 full-level workload (tensor + relin + rotate, "
                      "2 key switches each) "
                      "on synthetic residues, plain C oracle with OpenMP over limbs"}


def workload_config(cfg, batch: int, world: int, stored_a: bool = False, streams: str | None = None) -> dict:
    """The benchmark workload, the same for both arms."""
    c = {"workload": "n16-full: N=2^16, 36+12 primes < 2^30, dnum 3, level 35; "
                     f"step = batch of {batch} independent units, each tensor + relin + "
                     "rotate(1) with its own keys",
         "log_n": cfg.log_n, "n_q": cfg.n_q, "n_p": cfg.n_p, "dnum": cfg.dnum,
         "level": cfg.level, "batch": batch, "key_switches_per_step": KS_PER_UNIT * batch,
         "key_a_half": "stored (ablation)" if stored_a else "regenerated by ChaCha12",
         "l2": f"{N_SETS} rotating input/key sets (each > 126 MB L2)",
         "parallelism": f"replicas x{world}"}
    if streams:
        c["streams"] = streams
    return c


def run_reference(args, rank, world):
    if rank != 0:
        return
    one_step = _oracle_sample()
    for _ in range(args.warmup):
        one_step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one_step()
    dt = time.perf_counter() - t0
    value = KS_PER_UNIT * args.steps / dt
    cfg = W.CONFIGS[CONFIG_KEY]
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": "key-switches/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": 1e3 * dt / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "u32",
        "data": "synthetic",
        "config": workload_config(cfg, args.batch, world),
        "cpu_baseline": {"kind": "oracle", "cores": _omp_threads(), "value": value,
                         "unit": "key-switches/s",
                         "sample": f"{args.steps} timed steps, each a bounded sample of the workload: "
                                   f"1 of its {args.batch} units (tensor + relin + rotate, "
                                   f"{KS_PER_UNIT} key switches) on synthetic residues, plain C oracle "
                                   "with OpenMP over limbs on the host cores"},
        "e2e": {"value": value, "unit": "key-switches/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=8, help="independent n16-full units per step")
    ap.add_argument("--workload", default=CONFIG_KEY,
                    help="n16-full (benchmark line), or n16-bsgs32 / n16-stream64 / n16-stream64-rescale / "
                         "rescale / bsgs / bsgs-n14 (informational lines)")
    ap.add_argument("--streams", type=int, default=None,
                    help="CUDA streams the batch is split over, each running batch/streams units "
                         "(default 2 for an even batch, else 1)")
    ap.add_argument("--graph", action="store_true",
                    help="time one CUDA graph replay per step instead of eager launches (pays at small "
                         "batches; at 2 streams x 4 units the other stream already hides launch gaps)")
    ap.add_argument("--stored-a", action="store_true",
                    help="ablation: keys with a stored a half (read from HBM) instead of ChaCha12")
    args = ap.parse_args()
    rank, world, local_rank = rank_env()
    if args.impl == "reference":
        if args.steps > 3:
            args.steps = 3          # each oracle step is seconds of CPU work
        args.warmup = min(args.warmup, 1)
        run_reference(args, rank, world)
        return
    if str(args.workload) != CONFIG_KEY:
        run_workload(args, local_rank)
        return
    run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
