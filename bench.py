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
# workloads whose step is a batch of independent (tensor, relin, rotate) units: the benchmark line
# (n16-full) and informational lines on the N=2^12 chains
UNIT_WORKLOADS = ("n16-full", "n12-dnum2", "n12-dnum4")
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
    cfg = W.CONFIGS[args.workload]
    headline = args.workload == CONFIG_KEY
    n, lvl = cfg.n, cfg.level
    na = lvl + 1
    q, p = ks.ckks_gen_primes(cfg.log_n, cfg.n_q, cfg.n_p)
    ctx = ks.Context(cfg.log_n, q, p, cfg.dnum)
    set_bconv(ks, ctx, args)
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

    # the integer peaks of this GPU, measured now (a fraction of a second), for both rooflines
    peaks = measure_int_peaks(ks, dev)
    um = unit_model(cfg, lvl)
    cpu = cpu_baseline(args.workload) if (rank == 0 and world == 1 and not args.no_cpu_baseline) else None

    if rank == 0:
        line = {
            "metric": METRIC if headline else f"key-switches/s on {cfg.key} (informational)",
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
                           base_conversion=BCONV_ENGINES[args.bconv],
                           launch="one CUDA graph replay per step (captured per input set)" if graphs
                           else "eager launches"),
            "e2e": {"value": e2e_value, "unit": "key-switches/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": args.steps * LAUNCHES_PER_STEP * S,
            "kernel_launches_note": "one launch per kernel covers the whole batch",
            "clocks": clk,
            "roofline": roofline(cfg, dom_launches, dom_ms, clk, Bs, ms_single / args.steps,
                                 dom_launches_ov, dom_ms_ov, peaks),
            "path_roofline": dict(path_roofline(B * um["ops"], B * um["chacha_blocks"], B * um["bytes"],
                                                ms_per_step / 1e3, peaks),
                                  per="one step (the whole batch)"),
            "int_peaks": int_peaks_summary(peaks),
            "hbm_fraction_step": {"b_min_bytes_per_step": B * step_bytes_min(cfg),
                                  "frac": B * step_bytes_min(cfg) / (ms_per_step / 1e3) / (HBM_PEAK_GBS * 1e9),
                                  "peak_gbs": HBM_PEAK_GBS, "peak_source": PEAK_SOURCE},
            "cpu_baseline": cpu,
        }
        if not headline:
            line["informational"] = True
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
    """int32 issue ceiling, derived: 148 SMs x 4 sub-partitions x 32 lanes x 1 instruction/clock.
    Context only; the rooflines use the measured rates of `measure_int_peaks`."""
    return N_SM * 4 * 32 * mhz * 1e6 / 1e12


# ----------------------------------------------------------------------------- op model
# Algorithmic int32 operations of the path, with the unit costs of the op model: NTT butterfly 8
# (Shoup product 4, two lazy additions 2 + 2), constant modular product 4, modular addition 2,
# 32x32->64 multiply-add 2, 64->32 reduction 8, ChaCha12 block 608 (6 double rounds x 8
# quarter-rounds x 12 add/xor/rotate, plus 32 for the feed-forward and set-up; it yields 8
# coefficients), reduction of a 64-bit keystream word 8.
BFLY, CMUL, MADD, MAC, RED, CHACHA_BLOCK, AREDUCE = 8, 4, 2, 2, 8, 608, 8


def limb_ntt_ops(log_n: int) -> int:
    """One length-N negacyclic NTT (or inverse) of one limb: N/2 log N butterflies."""
    return (1 << log_n) // 2 * log_n * BFLY


def digit_sizes(cfg, level: int) -> list:
    na = level + 1
    return [min(cfg.alpha, na - lo) for lo in range(0, na, cfg.alpha)]


def modup_ops(cfg, level: int) -> int:
    """Inverse NTT of the l+1 limbs; per digit j (alpha_j primes) the base conversion onto the
    ext - alpha_j other limbs (alpha_j multiply-adds and one reduction per output) and their NTTs."""
    n, na = cfg.n, level + 1
    ext = na + cfg.n_p
    ds = digit_sizes(cfg, level)
    ntt = limb_ntt_ops(cfg.log_n)
    return na * ntt + sum((ext - a) * n * (a * MAC + RED) for a in ds) + sum(ext - a for a in ds) * ntt


def chacha_blocks(cfg, level: int) -> int:
    """ChaCha12 blocks that regenerate the a half of one key switch: beta * ext limbs of N/8."""
    na = level + 1
    return len(digit_sizes(cfg, level)) * (na + cfg.n_p) * cfg.n // 8


def ip_ops(cfg, level: int) -> int:
    """Key inner product: two multiply-adds per (digit, limb, coefficient), one reduction per
    accumulator word; plus the keystream's blocks and word reductions."""
    n, na = cfg.n, level + 1
    ext = na + cfg.n_p
    beta = len(digit_sizes(cfg, level))
    return (2 * beta * ext * n * MAC + 2 * ext * n * RED
            + chacha_blocks(cfg, level) * CHACHA_BLOCK + beta * ext * n * AREDUCE)


def moddown_ops(cfg, level: int, comps: int = 2) -> int:
    """Per component: inverse NTT of the k special limbs, base conversion P -> q_0..q_l, NTT of
    the l+1 converted limbs, (acc - conv) P^-1 (one product, one subtraction)."""
    n, na, k = cfg.n, level + 1, cfg.n_p
    ntt = limb_ntt_ops(cfg.log_n)
    return comps * (k * ntt + na * n * (k * MAC + RED) + na * ntt + na * n * (CMUL + MADD))


def keyswitch_ops(cfg, level: int) -> int:
    """One hybrid key switch (about 2.3 G at N=2^16, 36+12 primes, dnum 3, level 35)."""
    return modup_ops(cfg, level) + ip_ops(cfg, level) + moddown_ops(cfg, level)


def tensor_ops(cfg, level: int) -> int:
    """ct x ct: four products, one addition, three reductions per coefficient and limb."""
    return (level + 1) * cfg.n * (4 * MAC + 3 * RED)


def rescale_ops(cfg, level: int) -> int:
    """Per component: inverse NTT of limb l, NTT of its lift mod q_0..q_{l-1}, (c - conv) q_l^-1."""
    ntt = limb_ntt_ops(cfg.log_n)
    return 2 * (ntt + level * ntt + level * cfg.n * (CMUL + MADD))


def key_limbs(cfg, level: int) -> int:
    """Limbs of a key's b half one key switch reads: beta active digits x ext limbs."""
    return len(digit_sizes(cfg, level)) * (level + 1 + cfg.n_p)


def bsgs_level_model(cfg, lv: int, bg, gg):
    """One level of a slot DFT at level lv: the baby-step giant-step transform (one ModUp, the hoisted
    baby inner products, the plaintext sums in PQ, one ModDown per giant step, the giant rotations,
    the sum of the partials) and its rescale.  bg, gg: the Galois elements (1 = no rotation).
    Returns (op-model int32 operations, ChaCha12 blocks, compulsory bytes: input, plaintexts, the
    keys' b halves, output)."""
    n, limb = cfg.n, cfg.n * 4
    e_l, n_l = lv + 1 + cfg.n_p, lv + 1
    nb_r, ng_r = sum(g_ != 1 for g_ in bg), sum(g_ != 1 for g_ in gg)
    ops = (modup_ops(cfg, lv) + nb_r * ip_ops(cfg, lv) + len(gg) * len(bg) * 2 * e_l * n * MAC
           + len(gg) * 2 * e_l * n * RED + len(gg) * moddown_ops(cfg, lv)
           + ng_r * (keyswitch_ops(cfg, lv) + n_l * n * MADD) + len(gg) * 2 * n_l * n * MADD
           + rescale_ops(cfg, lv))
    blocks = (nb_r + ng_r) * chacha_blocks(cfg, lv)
    nbytes = ((len(gg) * len(bg) * e_l + 2 * n_l + 2 * n_l + 2 * n_l + 2 * (n_l - 1)) * limb
              + (nb_r + ng_r) * key_limbs(cfg, lv) * limb)
    return ops, blocks, nbytes


def evalmod_model(cfg, level: int, r: int, d: int, items: int):
    """EvalMod (degree 2d Taylor polynomial by Horner in theta^2, r double angles) on `items`
    ciphertexts that share the relinearisation key: (ops, ChaCha12 blocks, compulsory bytes: the
    key's b half once per product; inputs and outputs are counted by the caller).  The key's
    keystream is counted once per product, as the batched call regenerates it once."""
    n = cfg.n
    ops = blocks = nbytes = 0
    l = level

    def mult(l):
        # the items' relinearisations regenerate the key's a half once (they share one keystream)
        shared = (items - 1) * chacha_blocks(cfg, l) * CHACHA_BLOCK
        return (items * (tensor_ops(cfg, l) + keyswitch_ops(cfg, l) + 2 * (l + 1) * n * MADD + rescale_ops(cfg, l))
                - shared, chacha_blocks(cfg, l), key_limbs(cfg, l) * n * 4)

    def cmul_rescale(l):
        return items * (2 * (l + 1) * n * CMUL + rescale_ops(cfg, l))

    def addc(l):
        return items * (l + 1) * n * MADD
    ops += cmul_rescale(l) + addc(l - 1)                  # theta
    l -= 1
    for k in range(d + r):                                # theta^2, d - 1 Horner steps, r double angles
        if k == 1:                                        # the leading coefficient times u, rescale, + a_(d-1)
            ops += cmul_rescale(l) + addc(l - 1)
            l -= 1
        o, b, kb = mult(l)
        ops, blocks, nbytes = ops + o, blocks + b, nbytes + kb
        l -= 1
        if k > 0:                                         # + a_k, or (times 2) - 1 after a double angle
            ops += addc(l) + (items * 2 * (l + 1) * n * CMUL if k >= d else 0)
    ops += cmul_rescale(l)                                # times 1 / (2 pi)
    return ops, blocks, nbytes


def unit_model(cfg, level: int) -> dict:
    """One unit of the benchmark step (tensor, relinearisation, rotation): op-model int32 operations,
    ChaCha12 blocks and compulsory HBM bytes."""
    na, n = level + 1, cfg.n
    ops = tensor_ops(cfg, level) + 2 * keyswitch_ops(cfg, level) + 3 * na * n * MADD
    return {"ops": ops, "chacha_blocks": 2 * chacha_blocks(cfg, level), "bytes": step_bytes_min(cfg, level)}


def ip_row_ops(cfg) -> float:
    """Algorithmic int32 operations of one key switch's share of a k_ip_row8 launch, with the unit costs
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


# ----------------------------------------------------------------------------- measured int peaks
# Probes of ckks_int_probe (include/ckks_ks.h) and the iterations that make one launch last a few ms.
INT_PROBES = {"iadd": (0, 12288), "lop3": (1, 12288), "shf": (2, 12288), "imad": (3, 12288),
              "imad_hi": (4, 12288), "imad_wide": (5, 12288), "mix_lop3_imad": (6, 12288), "chacha12": (7, 1024)}
# the probes whose instruction any int32 operation of the op model can be issued as
GENERAL_PROBES = ("iadd", "lop3", "shf", "imad", "mix_lop3_imad")


def measure_int_peaks(ks, dev, reps: int = 3) -> dict:
    """Runs every probe `reps` times (after one warm-up launch) on all SMs and keeps the fastest:
    operations per second, per SM per clock (with the SM clock sampled meanwhile)."""
    import torch
    n_sms = torch.cuda.get_device_properties(dev).multi_processor_count
    blocks = n_sms * 6
    sink = torch.empty(blocks * 256, dtype=torch.uint32, device=dev)
    clocks = ClockSampler(dev.index or 0)
    clocks.start()
    time.sleep(0.2)
    res = {}
    for name, (op, iters) in INT_PROBES.items():
        ks.ckks_int_probe(op, blocks, iters, sink)                 # warm-up
        best = None
        for _ in range(reps):
            ms, ops = ks.ckks_int_probe(op, blocks, iters, sink)
            best = ms if best is None else min(best, ms)
        res[name] = {"ops_per_s": ops / (best / 1e3), "ms": best}
    clk = clocks.stop()
    mhz = clk.get("sm_mhz") or SM_MAX_MHZ
    for r in res.values():
        r["per_sm_per_clk"] = r["ops_per_s"] / (n_sms * mhz * 1e6)
    best_name = max(GENERAL_PROBES, key=lambda k: res[k]["ops_per_s"])
    return {"probes": res, "sm_mhz": mhz, "clocks": clk, "n_sms": n_sms,
            "int_tops": res[best_name]["ops_per_s"] / 1e12, "int_probe": best_name,
            "chacha_tops": res["chacha12"]["ops_per_s"] / 1e12,
            "source": f"measured live: ckks_int_probe, {blocks} blocks x 256 threads, 8 chains per thread, "
                      f"best of {reps}; int32 peak = fastest general probe ({best_name}); ChaCha12 peak = "
                      "the library's block function at 608 ops per block"}


def int_peaks_summary(peaks: dict) -> dict:
    """Compact record of the measured probes for the JSON line."""
    return {"sm_mhz": peaks["sm_mhz"], "int_tops": peaks["int_tops"], "int_probe": peaks["int_probe"],
            "chacha12_tops": peaks["chacha_tops"],
            "per_sm_per_clk": {k: round(v["per_sm_per_clk"], 2) for k, v in peaks["probes"].items()},
            "derived_issue_tops": alu_peak_tops(peaks["sm_mhz"])}


def _derived_peaks() -> dict:
    t = alu_peak_tops(SM_MAX_MHZ)
    return {"int_tops": t, "chacha_tops": t, "int_probe": None,
            "source": f"derived: {N_SM} SMs x 128 int32 lanes x {SM_MAX_MHZ:.0f} MHz (no measurement)"}


def int_time_s(ops: float, blocks: float, peaks: dict) -> float:
    """Time the op model's operations need at the measured peaks: every operation at the fastest
    general int32 rate, and the ChaCha12 blocks no faster than the measured ChaCha12 rate."""
    return max(ops / (peaks["int_tops"] * 1e12), blocks * CHACHA_BLOCK / (peaks["chacha_tops"] * 1e12))


def path_roofline(ops: float, blocks: float, nbytes: float, t_meas_s: float, peaks: dict) -> dict:
    """The whole path against the slower of its two floors: T_hbm = compulsory bytes / measured HBM
    bandwidth, T_int = op-model int32 operations at the measured integer peaks; frac = max / T."""
    t_int = int_time_s(ops, blocks, peaks)
    t_hbm = nbytes / (HBM_PEAK_GBS * 1e9)
    t_floor = max(t_int, t_hbm)
    return {"bound": "alu" if t_int >= t_hbm else "hbm", "frac": t_floor / t_meas_s,
            "t_measured_us": t_meas_s * 1e6, "t_int_us": t_int * 1e6, "t_hbm_us": t_hbm * 1e6,
            "int32_ops": ops, "chacha12_blocks": blocks, "hbm_bytes": nbytes,
            "int_peak_tops": peaks["int_tops"], "chacha12_peak_tops": peaks["chacha_tops"],
            "hbm_peak_gbs": HBM_PEAK_GBS, "hbm_frac": t_hbm / t_meas_s,
            "int_frac_at_general_peak": ops / (peaks["int_tops"] * 1e12) / t_meas_s,
            "peak_source": f"int: {peaks['source']}; hbm: {PEAK_SOURCE} (MEASURED_PEAKS.json copy)"
                           if PEAK_SOURCE == "measured" else f"int: {peaks['source']}; hbm: fallback 6650 GB/s"}


def roofline(cfg, launches, total_ms, clk, batch, single_step_ms, launches_ov, total_ms_ov, peaks=None):
    """The dominant kernel against its integer floor: achieved = algorithmic int32 operations per
    launch / average launch time; peak = the rate the measured peaks allow for this kernel's mix
    (its ChaCha12 blocks at the measured ChaCha12 rate, everything at the fastest general rate).
    `launches`/`total_ms`: its launches in a single-stream pass of the timed steps (each launch's
    events bracket that kernel only); `launches_ov`/`total_ms_ov`: the same kernel inside the timed
    multi-stream region, where its events also span the other streams' concurrent kernels."""
    if not launches:
        return None
    peaks = peaks or _derived_peaks()
    avg_s = total_ms / launches / 1e3
    ops = batch * ip_row_ops(cfg)
    blocks = batch * chacha_blocks(cfg, cfg.level)
    t_floor = int_time_s(ops, blocks, peaks)
    achieved = ops / avg_s / 1e12
    peak = ops / t_floor / 1e12
    traffic = ip_row_traffic_per_unit()
    out = {"kernel": "k_ip_row8 (ModUp last NTT pass + ChaCha12 + key inner product)",
           "bound": "alu", "achieved": achieved, "peak": peak, "unit": "Tops (int32)",
           "frac": achieved / peak,
           "traffic": None if traffic is None else traffic * batch,
           "units_per_launch": batch,
           "launches": launches,
           "avg_launch_us": avg_s * 1e6,
           "timed_in": "single-stream pass of the timed steps, right after the timed region "
                       f"({single_step_ms:.3f} ms per step)",
           "peak_source": peaks["source"],
           "frac_of_derived_issue_peak": achieved / alu_peak_tops(SM_MAX_MHZ)}
    if launches_ov:
        out["in_timed_region"] = {"launches": launches_ov,
                                  "avg_launch_us": total_ms_ov / launches_ov * 1e3,
                                  "note": "overlapped with the other streams' kernels"}
    return out


# DRAM bytes (read + write) per unit of a k_ip_row8 launch from an ncu capture, valid only for the
# kernel sources it was taken on (sha-256 prefix of the device-code headers): after any change to
# them the figure is reported as null until a new capture replaces it.
IP_ROW_TRAFFIC = {"sources_sha16": "93f7aa389dfb0d6d", "bytes_per_unit": (478.58e6 + 476.20e6) / 2 / 4,
                  "capture": "profiles/k_ip_row8_n16_full.md (dram__bytes read + write of two 4-unit launches)"}
KERNEL_HEADERS = ("debug_bounds.cuh", "modarith.cuh", "chacha.cuh", "ntt.cuh", "ks_kernels.cuh")


def kernel_sources_sha16() -> str:
    h = hashlib.sha256()
    for name in KERNEL_HEADERS:
        with open(os.path.join(ROOT, "fhe_key_switching_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ip_row_traffic_per_unit():
    if IP_ROW_TRAFFIC["sources_sha16"] != kernel_sources_sha16():
        return None
    return IP_ROW_TRAFFIC["bytes_per_unit"]


def step_bytes_min(cfg, level: int | None = None) -> int:
    """Compulsory HBM bytes of one unit: inputs, the keys' stored b halves and outputs of the
    tensor product (4 -> 3 polys), the relinearisation (3 polys + key -> 2) and the rotation
    (2 polys + key -> 2); the a halves are regenerated, intermediates are not counted."""
    level = cfg.level if level is None else level
    na = level + 1
    key = key_limbs(cfg, level)
    limbs = (4 + 3) * na + (3 * na + key + 2 * na) + (2 * na + key + 2 * na)
    return limbs * cfg.n * 4


# kernels launched by one step: tensor (1) + 2 key switches x 10 (ModUp 4, inner product with
# the last ModUp and first ModDown NTT passes 2, ModDown 4 including the fused combine)
LAUNCHES_PER_STEP = 1 + 2 * 10


def run_workload(args, local_rank):
    """Informational throughput (not the benchmark's headline line), each with its path roofline
    (op-model int32 operations and compulsory bytes against the measured peaks) and the oracle
    timed on a bounded sample of the same step:
    n14-hoisted8 = 8 units, each 8 hoisted rotations (+-1, +-2, +-4, +-8) of one ciphertext, then a
        tensor product and relinearisation with a second ciphertext (level 11, dnum 3);
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
    if key not in INFO_WORKLOADS:
        raise SystemExit(f"--workload {key}: use one of {', '.join(UNIT_WORKLOADS + INFO_WORKLOADS)}")
    cfg = W.CONFIGS[INFO_WORKLOADS[key]]
    n, lvl = cfg.n, cfg.level
    na = lvl + 1
    ext = na + cfg.n_p
    q, p = ks.ckks_gen_primes(cfg.log_n, cfg.n_q, cfg.n_p)
    ctx = ks.Context(cfg.log_n, q, p, cfg.dnum)
    set_bconv(ks, ctx, args)
    nd = -(-cfg.n_q // cfg.alpha)
    mods = q + p
    gen = W.rng(cfg.seed, W.TAG_SYNTH, 7)
    limb = n * 4

    def res(moduli):
        return torch.from_numpy(W.uniform_residues(moduli, n, gen)).to(dev)

    steps_g = sorted(set(cfg.rot_steps), key=cfg.rot_steps.index)
    gal = {r: ks.galois_element(cfg.log_n, r) for r in steps_g}
    keys_t = {r: res(mods * nd).view(nd, len(mods), n) for r in steps_g}
    evk = {r: ks.make_evk(keys_t[r], cfg.chacha_seed, gal[r]) for r in steps_g}
    stream = torch.cuda.current_stream(dev)
    ksw, kl = keyswitch_ops(cfg, lvl), key_limbs(cfg, lvl) * limb
    extra = {}
    if key == "n14-hoisted8":
        U, R = 8, len(cfg.rot_steps)
        cts = [res(q[:na] * 2 * U).view(U, 2, na, n) for _ in range(N_SETS)]
        ys = [res(q[:na] * 2 * U).view(U, 2, na, n) for _ in range(N_SETS)]
        k_rel = ks.make_evk(res(mods * nd).view(nd, len(mods), n), cfg.chacha_seed, 0)
        gs = [gal[r] for r in cfg.rot_steps]
        ev = [evk[r] for r in cfg.rot_steps]
        rot = torch.empty((U, R, 2, na, n), dtype=torch.uint32, device=dev)
        d = torch.empty((U, 3, na, n), dtype=torch.uint32, device=dev)
        rl = torch.empty((U, 2, na, n), dtype=torch.uint32, device=dev)
        ws_h = ctx.workspace(lvl, U * R, device=dev)
        ws_b = ctx.workspace(lvl, U, device=dev)

        def step(i):
            x, y = cts[i % N_SETS], ys[i % N_SETS]
            # the 8 units' hoisted rotations in one call: one ModUp per unit, one inner-product
            # launch over the 64 pairs, whose items with the same key share its keystream
            ks.ckks_rotate_hoisted_batch(ctx, x, lvl, gs, ev, rot, ws_h, stream)
            ks.ckks_tensor_batch(ctx, U, x, y, lvl, d, stream)
            ks.ckks_relin_batch(ctx, d, lvl, [k_rel] * U, rl, ws_b, stream)
        ks_per_step, rot_per_step = U * (R + 1), U * R
        # the units share the 8 rotation keys and the relinearisation key: their keystreams are
        # counted once per step, like their key bytes
        ops = (U * (modup_ops(cfg, lvl) + R * (ip_ops(cfg, lvl) + moddown_ops(cfg, lvl) + na * n * MADD)
                    + tensor_ops(cfg, lvl) + ksw + 2 * na * n * MADD)
               - (U - 1) * (R + 1) * chacha_blocks(cfg, lvl) * CHACHA_BLOCK)
        blocks = (R + 1) * chacha_blocks(cfg, lvl)
        nbytes = U * (2 * na * limb + R * 2 * na * limb + 7 * na * limb + 5 * na * limb) + (R + 1) * kl
    elif key == "n16-bsgs32":
        cts = [res(q[:na] * 2).view(2, na, n) for _ in range(N_SETS)]
        R = len(cfg.rot_steps)
        gs = [gal[r] for r in cfg.rot_steps]
        ev = [evk[r] for r in cfg.rot_steps]
        out = torch.empty((R, 2, na, n), dtype=torch.uint32, device=dev)
        ws = ctx.workspace(lvl, R, device=dev)

        def step(i):
            ks.ckks_rotate_hoisted(ctx, cts[i % N_SETS], lvl, gs, ev, out, ws, stream)
        ks_per_step, rot_per_step = R, R
        ops = modup_ops(cfg, lvl) + R * (ip_ops(cfg, lvl) + moddown_ops(cfg, lvl) + na * n * MADD)
        blocks = R * chacha_blocks(cfg, lvl)
        nbytes = 2 * na * limb + R * (kl + 2 * na * limb)
    elif key in ("n16-stream64", "n16-stream64-rescale"):
        rs = key.endswith("rescale")
        P_ = cfg.n_pairs
        lr = lvl - 1 if rs else lvl               # the rotation's level
        xs = [res(q[:na] * 2 * P_).view(P_, 2, na, n) for _ in range(2)]
        ys = [res(q[:na] * 2 * P_).view(P_, 2, na, n) for _ in range(2)]
        b_rel = res(mods * nd).view(nd, len(mods), n)
        k_rel = ks.make_evk(b_rel, cfg.chacha_seed, 0)
        d = torch.empty((P_, 3, na, n), dtype=torch.uint32, device=dev)
        r1 = torch.empty((P_, 2, na, n), dtype=torch.uint32, device=dev)
        r2 = torch.empty((P_, 2, lr + 1, n), dtype=torch.uint32, device=dev) if rs else r1
        out = torch.empty((P_, 2, lr + 1, n), dtype=torch.uint32, device=dev)
        ws = ctx.workspace(lvl, P_, device=dev)
        gs = [gal[r] for r in cfg.rot_steps]
        ev = [evk[r] for r in cfg.rot_steps]

        def step(i):
            ks.ckks_tensor_batch(ctx, P_, xs[i % 2], ys[i % 2], lvl, d, stream)
            ks.ckks_relin_batch(ctx, d, lvl, [k_rel] * P_, r1, ws, stream)
            if rs:
                ks.ckks_rescale_batch(ctx, P_, r1, lvl, r2, ws, stream)
            ks.ckks_rotate_batch(ctx, r2, lr, gs, ev, out, ws, stream)
        ks_per_step, rot_per_step = 2 * P_, P_
        nr = lr + 1
        # the keystreams counted once per distinct key and step (one relinearisation key, 15 rotation
        # keys), like the key bytes below: the items that share a key need its a half only once
        n_rk = len(set(gs))
        ops = (P_ * (tensor_ops(cfg, lvl) + ksw + 2 * na * n * MADD + keyswitch_ops(cfg, lr) + nr * n * MADD
                     + (rescale_ops(cfg, lvl) if rs else 0))
               - ((P_ - 1) * chacha_blocks(cfg, lvl) + (P_ - n_rk) * chacha_blocks(cfg, lr)) * CHACHA_BLOCK)
        blocks = chacha_blocks(cfg, lvl) + n_rk * chacha_blocks(cfg, lr)
        # per call, each key once (one relinearisation key, 15 rotation keys)
        nbytes = (P_ * (7 * na + 3 * na + 2 * na + (2 * na + 2 * nr if rs else 0) + 2 * nr + 2 * nr) * limb
                  + kl + len(steps_g) * key_limbs(cfg, lr) * limb)
    elif key == "rescale":
        R = 64
        cts = [res(q[:na] * 2 * R).view(R, 2, na, n) for _ in range(N_SETS)]
        out = torch.empty((R, 2, lvl, n), dtype=torch.uint32, device=dev)
        ws = ctx.workspace(lvl, R, device=dev)

        def step(i):
            ks.ckks_rescale_batch(ctx, R, cts[i % N_SETS], lvl, out, ws, stream)
        ks_per_step, rot_per_step = 0, 0
        ops, blocks = R * rescale_ops(cfg, lvl), 0
        nbytes = R * (2 * na + 2 * lvl) * limb
    elif key == "bootstrap":
        # one whole bootstrap per step (ckks_bootstrap) at N=2^16, dnum 4, levels 0 -> 35 -> 17: ModRaise
        # to level 35, CoeffToSlot (3 levels), the real/imaginary split (one conjugation), EvalMod on both
        # halves as one batch of two (degree 12, 3 double angles, 12 levels), the recombination,
        # SlotToCoeff (3 levels); synthetic plaintexts and keys (the cost is data independent)
        levels, n1, L = 3, 8, cfg.n_q - 1
        ns = n // 2
        halves_fwd = [1 << h for h in range(cfg.log_n - 2, -1, -1)]
        per = -(-len(halves_fwd) // levels)

        def dft_plan(top, inverse):
            hs_all = halves_fwd if inverse else halves_fwd[::-1]
            plan_ = []
            for li in range(levels):
                hs = hs_all[li * per:(li + 1) * per]
                st_ = min(hs)
                shifts = {0}
                for h in hs:
                    shifts = {((x_ + dd + ns // 2) % ns) - ns // 2 for x_ in shifts for dd in (-h, 0, h)}
                ms_ = sorted(x_ // st_ for x_ in shifts)
                bg_ = [1 if k == 0 else ks.galois_element(cfg.log_n, k * st_) for k in range(n1)]
                gg_ = [1 if g_ == 0 else ks.galois_element(cfg.log_n, g_ * n1 * st_)
                       for g_ in range(ms_[0] // n1, ms_[-1] // n1 + 1)]
                lv_ = top - li
                pt_ = res((q[:lv_ + 1] + p) * len(gg_) * len(bg_)).view(len(gg_), len(bg_), lv_ + 1 + cfg.n_p, n)
                plan_.append((lv_, bg_, gg_, pt_, None))
            return plan_
        c2s, s2c = dft_plan(L, True), dft_plan(L - 3 - 12, False)
        gk = {}
        for _, bg_, gg_, _, _ in c2s + s2c:
            for g_ in bg_ + gg_:
                if g_ != 1 and g_ not in gk:
                    gk[g_] = ks.make_evk(res(mods * nd).view(nd, len(mods), n), cfg.chacha_seed, g_)
        gconj = ks.conjugation_element(cfg.log_n)
        k_conj = ks.make_evk(res(mods * nd).view(nd, len(mods), n), cfg.chacha_seed, gconj)
        k_rel = ks.make_evk(res(mods * nd).view(nd, len(mods), n), cfg.chacha_seed, 0)
        cts0 = [res(q[:1] * 2).view(2, 1, n) for _ in range(N_SETS)]

        def plan_levels(plan_):
            return [(bg_, [gk.get(g_) for g_ in bg_], gg_, [gk.get(g_) for g_ in gg_], pt_)
                    for _, bg_, gg_, pt_, _ in plan_]
        bplan = ks.BootstrapPlan(L, plan_levels(c2s), plan_levels(s2c), k_conj, k_rel, 3, 6)
        ws_bt = ks.ckks_bootstrap_workspace(ctx, bplan, device=dev)
        out = torch.empty((2, bplan.out_level + 1, n), dtype=torch.uint32, device=dev)

        def step(i):
            ks.ckks_bootstrap(ctx, cts0[i % N_SETS], bplan, out, ws_bt, stream)
        # the transforms' rotations and the conjugation, plus EvalMod's d + r relinearisations per half
        rot_per_step = sum(sum(1 for g_ in bg_ + gg_ if g_ != 1) for _, bg_, gg_, _, _ in c2s + s2c) + 1
        ks_per_step = rot_per_step + 2 * (6 + 3)
        # op model: ModRaise (inverse NTT of limb 0, lift and NTT into 36 limbs, both components),
        # the six DFT levels, the conjugation, the split and the recombination, EvalMod on both
        # halves; compulsory bytes: the input, plaintexts and keys (the levels' and EvalMod's), output
        lz, lo = L - levels, L - levels - 12
        ntt1 = limb_ntt_ops(cfg.log_n)
        ops = 2 * (ntt1 + (L + 1) * (n * RED + ntt1))
        blocks = 0
        nbytes = 2 * limb + 2 * (bplan.out_level + 1) * limb + key_limbs(cfg, lz) * limb
        for lv_, bg_, gg_, _, _ in c2s + s2c:
            o_, b_, _ = bsgs_level_model(cfg, lv_, bg_, gg_)
            ops, blocks = ops + o_, blocks + b_
            nbytes += (len(gg_) * len(bg_) * (lv_ + 1 + cfg.n_p)
                       + sum(g_ != 1 for g_ in bg_ + gg_) * key_limbs(cfg, lv_)) * limb
        ops += keyswitch_ops(cfg, lz) + (lz + 1) * n * MADD + 2 * (lz + 1) * n * (2 * MADD + CMUL)
        blocks += chacha_blocks(cfg, lz)
        o_, b_, n_ = evalmod_model(cfg, lz, 3, 6, 2)
        ops, blocks, nbytes = ops + o_ + 2 * (lo + 1) * n * (MADD + CMUL), blocks + b_, nbytes + n_
        extra["_boot_level"] = (c2s[0][0], c2s[0][1], c2s[0][2])
    elif key == "coeff-to-slot":
        # CoeffToSlot of N=2^16 in 3 levels of 5 radix-2 stages: each level's 63 slot diagonals
        # (shifts m s, |m| <= 31, s its smallest half-length) as 8 baby x 8 giant steps, then a
        # rescale; plaintexts and keys are synthetic residues (the cost is data independent)
        levels, n1 = 3, 8
        ns = n // 2
        halves = [1 << h for h in range(cfg.log_n - 2, -1, -1)]          # n/4 ... 1, applied in order
        per = -(-len(halves) // levels)
        steps = [min(halves[i:i + per]) for i in range(0, len(halves), per)]
        plan, gk = [], {}
        for li, st_ in enumerate(steps):
            lv = lvl - li
            # the level's shifts: signed sums of its stages' half-lengths, centred in [-n/2, n/2)
            shifts = {0}
            for h in halves[li * per:(li + 1) * per]:
                shifts = {((x + d + ns // 2) % ns) - ns // 2 for x in shifts for d in (-h, 0, h)}
            ms = sorted(x // st_ for x in shifts)
            babies = [k * st_ for k in range(n1)]
            giants = [g * n1 * st_ for g in range(ms[0] // n1, ms[-1] // n1 + 1)]
            bg = [1 if b % ns == 0 else ks.galois_element(cfg.log_n, b) for b in babies]
            gg = [1 if g_ % ns == 0 else ks.galois_element(cfg.log_n, g_) for g_ in giants]
            for g_ in bg + gg:
                if g_ != 1 and g_ not in gk:
                    gk[g_] = ks.make_evk(res(mods * nd).view(nd, len(mods), n), cfg.chacha_seed, g_)
            ext_l = lv + 1 + cfg.n_p
            pt_l = res((q[:lv + 1] + p) * len(gg) * len(bg)).view(len(gg), len(bg), ext_l, n)
            plan.append((lv, bg, gg, pt_l, ks.ckks_bsgs_workspace(ctx, lv, len(bg), len(gg), device=dev)))
        cts = [res(q[:na] * 2).view(2, na, n) for _ in range(N_SETS)]
        mids = [torch.empty((2, lv + 1, n), dtype=torch.uint32, device=dev) for lv, *_ in plan]
        outs = [torch.empty((2, lv, n), dtype=torch.uint32, device=dev) for lv, *_ in plan]
        ws_r = ctx.workspace(lvl, 1, device=dev)

        def step(i):
            cur = cts[i % N_SETS]
            for (lv, bg, gg, pt_l, ws_l), mid, o in zip(plan, mids, outs):
                ks.ckks_bsgs(ctx, cur, lv, bg, [gk.get(g_) for g_ in bg], gg, [gk.get(g_) for g_ in gg], pt_l,
                             mid, ws_l, stream)
                ks.ckks_rescale(ctx, mid, lv, o, ws_r, stream)
                cur = o
        ks_per_step = rot_per_step = sum(sum(1 for g_ in bg + gg if g_ != 1) for _, bg, gg, _, _ in plan)
        ops = blocks = nbytes = 0
        for lv, bg, gg, pt_l, _ in plan:
            o_, b_, n_ = bsgs_level_model(cfg, lv, bg, gg)
            ops, blocks, nbytes = ops + o_, blocks + b_, nbytes + n_
    else:                                          # bsgs, bsgs-n14
        n1, n2 = 16, 18
        baby = [1] + [ks.galois_element(cfg.log_n, k) for k in range(1, n1)]
        giant = [1] + [ks.galois_element(cfg.log_n, n1 * j) for j in range(1, n2)]
        gk = {g: ks.make_evk(res(mods * nd).view(nd, len(mods), n), cfg.chacha_seed, g)
              for g in baby + giant if g != 1}
        pt = res((q[:na] + p) * n2 * n1).view(n2, n1, ext, n)
        cts = [res(q[:na] * 2).view(2, na, n) for _ in range(N_SETS)]
        out = torch.empty((2, na, n), dtype=torch.uint32, device=dev)
        ws = ks.ckks_bsgs_workspace(ctx, lvl, n1, n2, device=dev)
        bk = [gk.get(g) for g in baby]
        gkk = [gk.get(g) for g in giant]

        def step(i):
            ks.ckks_bsgs(ctx, cts[i % N_SETS], lvl, baby, bk, giant, gkk, pt, out, ws, stream)
        ks_per_step, rot_per_step = (n1 - 1) + (n2 - 1), (n1 - 1) + (n2 - 1)
        # one ModUp, 15 hoisted inner products, the plaintext sums (two multiply-adds and a
        # reduction share per term), 18 ModDowns, 17 giant rotations, the sum of 18 partials
        ops = (modup_ops(cfg, lvl) + (n1 - 1) * ip_ops(cfg, lvl) + n2 * n1 * 2 * ext * n * MAC
               + n2 * 2 * ext * n * RED + n2 * moddown_ops(cfg, lvl) + (n2 - 1) * (ksw + na * n * MADD)
               + n2 * 2 * na * n * MADD)
        blocks = (n1 - 1 + n2 - 1) * chacha_blocks(cfg, lvl)
        nbytes = (n2 * n1 * ext + 2 * na + 2 * na) * limb + (n1 - 1 + n2 - 1) * kl
        b_comb = (n2 * n1 * ext + (n1 - 1) * 2 * ext + 2 * na + n2 * 2 * ext) * limb
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    is_bsgs = key in ("bsgs", "bsgs-n14")
    if is_bsgs:
        ks.ckks_prof_begin(ctx, "bsgs_combine", args.steps)
    e0.record(stream)
    for i in range(args.steps):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    if is_bsgs:
        launches, comb_ms = ks.ckks_prof_end(ctx)
        comb_s = comb_ms / max(launches, 1) / 1e3
        extra["combine_kernel"] = {"avg_launch_us": comb_s * 1e6, "launches": launches,
                                   "bytes_per_launch": b_comb, "achieved_gbs": b_comb / comb_s / 1e9,
                                   "peak_gbs": HBM_PEAK_GBS, "frac": b_comb / comb_s / 1e9 / HBM_PEAK_GBS,
                                   "share_of_step": comb_s * 1e3 / (ms / args.steps)}
    peaks = measure_int_peaks(ks, dev)
    t_step = ms / args.steps / 1e3
    line = {"workload": key, "informational": True, "config": INFO_DESCRIPTIONS[key],
            "base_conversion": BCONV_ENGINES[args.bconv],
            "ms_per_step": ms / args.steps, "steps": args.steps, "warmup": args.warmup}
    if key == "rescale":
        line["rescales_per_s"] = R / t_step
    elif key == "bootstrap":
        line["ms_per_bootstrap"] = t_step * 1e3
        line["context"] = ("the EncryptedLLM summary (lpnh.cn page, Results) quotes 22-27 ms per bootstrap on an "
                           "unnamed GPU with its own parameters; context only, not a target")
    elif key == "coeff-to-slot":
        line["ms_per_coeff_to_slot"] = t_step * 1e3
        line["context"] = ("the EncryptedLLM summary (lpnh.cn page, Results) quotes 22-27 ms per whole "
                           "bootstrap on an unnamed GPU; CoeffToSlot is one of its three parts")
    elif is_bsgs:
        line["transforms_per_s"] = 1 / t_step
        line["rotations_per_transform"] = rot_per_step
    if ks_per_step:
        line["key_switches_per_s"] = ks_per_step / t_step
        line["rotations_per_s"] = rot_per_step / t_step
        line["key_switches_per_step"] = ks_per_step
    if ops:
        line["path_roofline"] = dict(path_roofline(ops, blocks, nbytes, t_step, peaks), per="one step")
    boot_level = extra.pop("_boot_level", None)
    line.update(extra)
    line["int_peaks"] = int_peaks_summary(peaks)
    line["clocks"] = clk
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = info_cpu_baseline(key, ops_step=ops, boot_level=boot_level)
    print(json.dumps(line), flush=True)


INFO_WORKLOADS = {"coeff-to-slot": "n16-bsgs32", "bootstrap": "n16-stream64",
                  "n14-hoisted8": "n14-hoisted8", "n16-bsgs32": "n16-bsgs32", "n16-stream64": "n16-stream64",
                  "n16-stream64-rescale": "n16-stream64", "rescale": "n16-full", "bsgs": "n16-bsgs32",
                  "bsgs-n14": "n14-hoisted8"}
INFO_DESCRIPTIONS = {
    "bootstrap": "N=2^16, 36+12 primes, dnum 4; step = one ckks_bootstrap from level 0: ModRaise to level 35, "
                 "CoeffToSlot (3 levels), the real/imaginary split (a conjugation), EvalMod on both halves (12 "
                 "levels, degree 12, 3 double angles), the recombination, SlotToCoeff (3 levels), output at level 17",
    "coeff-to-slot": "N=2^16, 36+12 primes, dnum 4, from level 24; step = CoeffToSlot in 3 levels of 5 radix-2 "
                     "stages, each an 8 baby x 8 giant step transform of 63 slot diagonals plus a rescale",
    "n14-hoisted8": "N=2^14, 12+4 primes, dnum 3, level 11; step = 8 units, each 8 hoisted rotations "
                    "(+-1, +-2, +-4, +-8) + tensor + relin; the units' rotations as one ckks_rotate_hoisted_batch call",
    "n16-bsgs32": "N=2^16, 36+12 primes, dnum 4, level 24; step = 32 hoisted rotations of one ciphertext",
    "n16-stream64": "N=2^16, 36+12 primes, dnum 4, level 20; step = 64 pairs, each tensor + relin + "
                    "rotate by 2^(i mod 15)",
    "n16-stream64-rescale": "as n16-stream64 with a rescale after the relinearisation (rotation at level 19)",
    "rescale": "N=2^16, 36+12 primes, level 35 -> 34; step = 64 rescales",
    "bsgs": "N=2^16, 36+12 primes, dnum 4, level 24; step = one 16 baby x 18 giant step transform "
            "(288 plaintext diagonals)",
    "bsgs-n14": "N=2^14, 12+4 primes, dnum 3, level 11; step = one 16 baby x 18 giant step transform",
}


def info_cpu_baseline(key: str, max_seconds: float = 8.0, ops_step: float = 0.0, boot_level=None):
    """The oracle on a bounded sample of an informational line's step (synthetic residues; the cost
    is data independent), in the line's own unit.  For the whole bootstrap the sample is its first
    CoeffToSlot level (boot_level: its level and Galois elements) and one EvalMod half, and the
    step's time is estimated from the sample by the op model (ops_step: the step's count)."""
    import numpy as np
    import oracle

    cfg = W.CONFIGS[INFO_WORKLOADS[key]]
    n, lvl = cfg.n, cfg.level
    na = lvl + 1
    octx = oracle.Ctx(cfg.log_n, cfg.n_q, cfg.n_p)
    nd = -(-cfg.n_q // cfg.alpha)
    gen = W.rng(cfg.seed, W.TAG_SYNTH, 98)
    ct = W.uniform_residues(octx.q[:na] * 2, n, gen).reshape(2, na, n)
    b = W.uniform_residues(octx.mod * nd, n, gen).reshape(nd, len(octx.mod), n)
    seed = cfg.chacha_seed
    if key == "bootstrap":
        from oracle import bootstrap as obt
        lz = cfg.n_q - 1 - 3                            # EvalMod's input level in the bootstrap
        ctz = W.uniform_residues(octx.q[:lz + 1] * 2, n, gen).reshape(2, lz + 1, n)
        lv, bg, gg = boot_level
        ct_l = W.uniform_residues(octx.q[:lv + 1] * 2, n, gen).reshape(2, lv + 1, n)
        ext_l = lv + 1 + cfg.n_p
        pt = W.uniform_residues((octx.q[:lv + 1] + octx.p) * len(gg) * len(bg), n, gen).reshape(
            len(gg), len(bg), ext_l, n)
        bk = [None if g_ == 1 else (b, g_) for g_ in bg]
        gk = [None if g_ == 1 else (b, g_) for g_ in gg]
        t0 = time.perf_counter()
        octx.rescale(octx.bsgs(ct_l, lv, cfg.alpha, bg, bk, gg, gk, pt, seed), lv)
        obt.evalmod(octx, ctz, lz, float(octx.q[0]), 3, 6, cfg.alpha, b, seed)
        dt = time.perf_counter() - t0
        ratio = ops_step / (evalmod_model(cfg, lz, 3, 6, 1)[0] + bsgs_level_model(cfg, lv, bg, gg)[0])
        return {"value": dt * ratio * 1e3, "unit": "ms per bootstrap (estimate)", "cores": _omp_threads(),
                "kind": "oracle",
                "sample": f"the first CoeffToSlot level (level {lv}, {len(bg)} baby x {len(gg)} giant steps, "
                          f"rescale) and one EvalMod half (9 products, level {lz} -> {lz - 12}) on synthetic "
                          f"residues, {dt:.2f} s, scaled by the op model's ratio of the whole bootstrap to them "
                          f"({ratio:.2f}); plain C oracle with OpenMP over limbs"}
    if key in ("bsgs", "coeff-to-slot"):
        return None                 # the oracle's plaintext sums take minutes at N=2^16
    if key == "n14-hoisted8":
        gs = [octx.galois(r) for r in cfg.rot_steps]
        y = W.uniform_residues(octx.q[:na] * 2, n, gen).reshape(2, na, n)

        def fn():
            octx.rotate_hoisted(ct, lvl, cfg.alpha, gs, [b] * len(gs), [seed] * len(gs), gs)
            octx.relin(octx.tensor(ct, y, lvl), lvl, cfg.alpha, b, seed, 0)
        units, unit, what = len(gs) + 1, "key-switches/s", "one unit (8 hoisted rotations + tensor + relin)"
    elif key == "n16-bsgs32":
        gs = [octx.galois(r) for r in cfg.rot_steps[:2]]

        def fn():
            octx.rotate_hoisted(ct, lvl, cfg.alpha, gs, [b] * 2, [seed] * 2, gs)
        units, unit, what = 2, "rotations/s", "2 of the 32 hoisted rotations (one ModUp)"
    elif key in ("n16-stream64", "n16-stream64-rescale"):
        y = W.uniform_residues(octx.q[:na] * 2, n, gen).reshape(2, na, n)
        g = octx.galois(1)

        def fn():
            r = octx.relin(octx.tensor(ct, y, lvl), lvl, cfg.alpha, b, seed, 0)
            lv = lvl
            if key.endswith("rescale"):
                r, lv = octx.rescale(r, lvl), lvl - 1
            octx.rotate(r, lv, cfg.alpha, g, b, seed, g)
        units, unit, what = 2, "key-switches/s", "one pair of the 64"
    elif key == "rescale":
        def fn():
            octx.rescale(ct, lvl)
        units, unit, what = 1, "rescales/s", "one of the 64 rescales"
    else:                           # bsgs-n14
        n1, n2 = 16, 18
        ext = na + cfg.n_p
        baby = [1] + [octx.galois(k) for k in range(1, n1)]
        giant = [1] + [octx.galois(n1 * j) for j in range(1, n2)]
        pt = W.uniform_residues((octx.q[:na] + octx.p) * n1 * n2, n, gen).reshape(n2, n1, ext, n)
        kb = [None] + [(b, g) for g in baby[1:]]
        kg = [None] + [(b, g) for g in giant[1:]]

        def fn():
            octx.bsgs(ct, lvl, cfg.alpha, baby, kb, giant, kg, pt, seed)
        units, unit, what = 1, "transforms/s", "one whole transform"
    fn()
    t0 = time.perf_counter()
    k = 0
    while True:
        fn()
        k += 1
        if time.perf_counter() - t0 > max_seconds / 2 or k >= 16:
            break
    dt = time.perf_counter() - t0
    return {"value": units * k / dt, "unit": unit, "cores": _omp_threads(), "kind": "oracle",
            "sample": f"{k} x {what} of {key} on synthetic residues, plain C oracle with OpenMP over limbs"}


BCONV_ENGINES = {"cuda": "CUDA cores (32x32->64-bit multiply-adds)",
                 "tensor": "tensor cores (8-bit split, tcgen05.mma kind::i8)",
                 "auto": "automatic: tensor cores (8-bit split, tcgen05.mma kind::i8) for launches of at least "
                         "4 tiles per block, CUDA cores below"}


def set_bconv(ks, ctx, args):
    ks.ckks_set_bconv_mode(ctx, {"tensor": ks.CKKS_BCONV_TENSOR, "cuda": ks.CKKS_BCONV_CUDA_CORES,
                                 "auto": ks.CKKS_BCONV_AUTO}[args.bconv])


def run_int_peaks(local_rank):
    """Informational line: the integer probes of ckks_int_probe, as operations per second and per
    SM per clock at the sampled SM clock."""
    import torch
    import fhe_key_switching_b200 as ks
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    peaks = measure_int_peaks(ks, dev, reps=5)
    print(json.dumps({"informational": True, "int_peaks": {
        k: {"tops": v["ops_per_s"] / 1e12, "per_sm_per_clk": v["per_sm_per_clk"], "ms": v["ms"]}
        for k, v in peaks["probes"].items()},
        "sm_mhz": peaks["sm_mhz"], "n_sms": peaks["n_sms"], "int_tops": peaks["int_tops"],
        "int_probe": peaks["int_probe"], "chacha12_tops": peaks["chacha_tops"],
        "derived_issue_tops": alu_peak_tops(peaks["sm_mhz"]), "source": peaks["source"],
        "clocks": peaks["clocks"]}), flush=True)


def _oracle_sample(key: str = CONFIG_KEY):
    """Bounded CPU sample of the same step: one unit (tensor, relinearisation, rotation) of the
    workload, timed on the oracle with synthetic residues (cost is data independent)."""
    import numpy as np
    import oracle

    cfg = W.CONFIGS[key]
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


def cpu_baseline(key: str = CONFIG_KEY, max_seconds: float = 20.0):
    one_step = _oracle_sample(key)
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
            "sample": f"{k} units of the {key} workload (tensor + relin + rotate, 2 key switches each) "
                      "on synthetic residues, plain C oracle with OpenMP over limbs"}


def workload_config(cfg, batch: int, world: int, stored_a: bool = False, streams: str | None = None) -> dict:
    """The benchmark workload, the same for both arms."""
    c = {"workload": f"{cfg.key}: N=2^{cfg.log_n}, {cfg.n_q}+{cfg.n_p} primes < 2^30, dnum {cfg.dnum}, "
                     f"level {cfg.level}; step = batch of {batch} independent units, each tensor + relin + "
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
    ap.add_argument("--batch", type=int, default=None,
                    help="independent units per step (default 8 for n16-full, 64 for the N=2^12 lines)")
    ap.add_argument("--workload", default=CONFIG_KEY,
                    help="n16-full (benchmark line), or n12-dnum2 / n12-dnum4 / n14-hoisted8 / n16-bsgs32 / "
                         "n16-stream64 / n16-stream64-rescale / rescale / bsgs / bsgs-n14 / coeff-to-slot / bootstrap "
                         "(informational lines)")
    ap.add_argument("--streams", type=int, default=None,
                    help="CUDA streams the batch is split over, each running batch/streams units "
                         "(default 2 for an even batch, else 1)")
    ap.add_argument("--graph", action="store_true",
                    help="time one CUDA graph replay per step instead of eager launches (pays at small "
                         "batches; at 2 streams x 4 units the other stream already hides launch gaps)")
    ap.add_argument("--bconv", default="auto", choices=sorted(BCONV_ENGINES),
                    help="base-conversion engine: auto (default: tensor cores for large launches), tensor "
                         "(8-bit split on the tensor cores) or cuda (CUDA cores); the output bits are the same")
    ap.add_argument("--int-peaks", action="store_true",
                    help="measure this GPU's integer throughput per instruction class (ckks_int_probe) and "
                         "print it as one JSON line")
    ap.add_argument("--stored-a", action="store_true",
                    help="ablation: keys with a stored a half (read from HBM) instead of ChaCha12")
    args = ap.parse_args()
    rank, world, local_rank = rank_env()
    if args.batch is None:
        args.batch = 8 if args.workload == CONFIG_KEY or args.impl == "reference" else 64
    if args.impl == "reference":
        if args.steps > 3:
            args.steps = 3          # each oracle step is seconds of CPU work
        args.warmup = min(args.warmup, 1)
        run_reference(args, rank, world)
        return
    if args.int_peaks:
        run_int_peaks(local_rank)
        return
    if str(args.workload) not in UNIT_WORKLOADS:
        run_workload(args, local_rank)
        return
    run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
