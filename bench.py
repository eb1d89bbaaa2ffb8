"""Benchmark of the MALA hot path on B200.

One step = the whole hot path on one batch of synthetic input:
  * long-context training operator, B=1 H=8 L=131072 d=128 bf16, tile 128,
    tau=1: mala_fwd then mala_bwd;
  * long-context decode, B=16 Hq=32 Hkv=8 Lc=131072 d=128 bf16 cache, tau=1:
    one mala_decode step.
The metric is milliseconds per step (lower is better), with the per-call
breakdown (fwd ms, bwd ms, decode us), effective TFLOP/s (full legal QK plus
retained post-score work), retained slots per query and the roofline fraction
of the dominant kernel. The same kernels at tau=0 (dense) are timed beside it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mala|reference]

N > 1 runs under torchrun, one rank per GPU; the work shards by (batch, head)
with no exchange step, so every rank runs its own independent copy of the
workload (weak scaling) and rank 0 prints the max-over-ranks time.
Inputs are larger than L2 (805 MB of Q/K/V per prefill pass, 8.6 GB of KV
cache), so no flush is needed between steps.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

PREFILL = synth.CONFIGS["long_128k"]
DECODE = synth.CONFIGS["decode_128k"]
WORKLOAD = "long_128k fwd+bwd (B1 H8 L131072 d128 bf16 tile128 tau=1) + decode_128k (B16 Hq32 Hkv8 Lc131072 d128 bf16 tau=1)"


# ---------------------------------------------------------------------------
# input generation (host, numpy; parallel over sequences with a spawn pool)
# ---------------------------------------------------------------------------
def _bf16_bits(a: np.ndarray) -> np.ndarray:
    """float64 -> bf16 bit patterns (round to nearest even) as uint16."""
    f = a.astype(np.float32)
    u = f.view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> 16) & np.uint32(1))) >> 16
    return r.astype(np.uint16)


def _gen_prefill_seq(args):
    cfg_name, s, shm_names, L, d, seed_shift = args
    from multiprocessing import shared_memory
    cfg = synth.CONFIGS[cfg_name]
    seq = synth.prefill_sequence(cfg.config_seed + seed_shift, s, L, d, cfg.rho, cfg.n_pairs)
    for n, shm_name in shm_names.items():
        shm = shared_memory.SharedMemory(name=shm_name)
        arr = np.ndarray((cfg.B * cfg.H, L, d), dtype=np.uint16, buffer=shm.buf)
        arr[s] = _bf16_bits(seq[n])
        del arr
        shm.close()
    return s


def _gen_decode_group(args):
    s, shm_names, seed_shift = args
    from multiprocessing import shared_memory
    cfg = DECODE
    if seed_shift:
        cfg = synth.DecodeConfig(cfg.name, cfg.config_seed + seed_shift, cfg.B, cfg.Hq, cfg.Hkv,
                                 cfg.Lc, cfg.d, cfg.tile, cfg.rho, cfg.n_pairs, cfg.n_query_targets)
    b, g = divmod(s, cfg.Hkv)
    grp = synth.decode_group(cfg, b, g)
    G = cfg.Hq // cfg.Hkv
    for n in ("K", "V"):
        shm = shared_memory.SharedMemory(name=shm_names[n])
        arr = np.ndarray((cfg.B * cfg.Hkv, cfg.Lc, cfg.d), dtype=np.uint16, buffer=shm.buf)
        arr[s] = _bf16_bits(grp[n])
        del arr
        shm.close()
    shm = shared_memory.SharedMemory(name=shm_names["q"])
    arr = np.ndarray((cfg.B * cfg.Hkv, G, cfg.d), dtype=np.uint16, buffer=shm.buf)
    arr[s] = _bf16_bits(grp["q"])
    del arr
    shm.close()
    return s


def generate_inputs(workers: int, seed_shift: int = 0):
    """Returns dict of uint16 (bf16 bit) numpy arrays; runs before any CUDA
    call so the spawn pool is safe."""
    import multiprocessing as mp
    from multiprocessing import shared_memory
    ctx = mp.get_context("spawn")
    P = PREFILL
    shapes = {n: (P.B * P.H, P.L, P.d) for n in ("Q", "K", "V", "dO")}
    G = DECODE.Hq // DECODE.Hkv
    dshapes = {"K": (DECODE.B * DECODE.Hkv, DECODE.Lc, DECODE.d),
               "V": (DECODE.B * DECODE.Hkv, DECODE.Lc, DECODE.d),
               "q": (DECODE.B * DECODE.Hkv, G, DECODE.d)}
    shms = {}
    try:
        for n, shp in shapes.items():
            shms["p" + n] = shared_memory.SharedMemory(create=True, size=int(np.prod(shp)) * 2)
        for n, shp in dshapes.items():
            shms["d" + n] = shared_memory.SharedMemory(create=True, size=int(np.prod(shp)) * 2)
        pre_names = {n: shms["p" + n].name for n in shapes}
        dec_names = {n: shms["d" + n].name for n in dshapes}
        jobs_p = [(P.name, s, pre_names, P.L, P.d, seed_shift) for s in range(P.B * P.H)]
        jobs_d = [(s, dec_names, seed_shift) for s in range(DECODE.B * DECODE.Hkv)]
        with ctx.Pool(max(1, workers)) as pool:
            pool.map(_gen_prefill_seq, jobs_p)
            pool.map(_gen_decode_group, jobs_d)
        out = {}
        for n, shp in shapes.items():
            out["p" + n] = np.ndarray(shp, dtype=np.uint16, buffer=shms["p" + n].buf).copy()
        for n, shp in dshapes.items():
            out["d" + n] = np.ndarray(shp, dtype=np.uint16, buffer=shms["d" + n].buf).copy()
        return out
    finally:
        for s in shms.values():
            s.close()
            s.unlink()


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi sampling of one GPU's SM clock and throttle reasons.

    start() launches the sampler and waits (at most a few seconds) until it
    has written a first sample, so that the timed region that follows is
    covered; mark("begin") / mark("end") bracket the timed region on the
    host clock; stop() summarises the samples whose timestamps fall inside
    that window (all samples when none does, and the line says which).
    Throttle reasons are collected over every sample of the run."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,"
              "timestamp")
    PERIOD_MS = 50
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index: int, tool: str = "nvidia-smi"):
        self.gpu = gpu_index
        self.tool = tool
        self.proc = None
        self.marks = {}
        # the raw samples go to MALA_BENCH_OUT (default: the system's temp
        # directory); the JSON line carries their summary
        import tempfile
        out = os.environ.get("MALA_BENCH_OUT", tempfile.gettempdir())
        self.path = os.path.join(out, f"clocks_gpu{gpu_index}.csv")

    def start(self, first_sample_timeout: float = 3.0):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                [self.tool, "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", str(self.PERIOD_MS)], stdout=self.fh,
                stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            return
        t0 = time.time()
        while time.time() - t0 < first_sample_timeout and self.proc.poll() is None:
            try:
                if os.path.getsize(self.path) > 0:
                    break
            except OSError:
                break
            time.sleep(0.01)

    def mark(self, which: str):
        import datetime
        self.marks[which] = datetime.datetime.now()

    @staticmethod
    def _timestamp(text: str):
        import datetime
        for fmt in ("%Y/%m/%d %H:%M:%S.%f", "%Y/%m/%d %H:%M:%S"):
            try:
                return datetime.datetime.strptime(text, fmt)
            except ValueError:
                pass
        return None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        rows, reasons = [], set()
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm, smax = float(f[1]), float(f[2])
            except ValueError:
                continue
            for n, v in zip(self.REASONS, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
            rows.append((self._timestamp(f[9]) if len(f) > 9 else None, sm, smax))
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        import datetime
        b, e = self.marks.get("begin"), self.marks.get("end")
        inside = []
        if b is not None and e is not None:
            # a sample stands for the period that ends at its timestamp
            late = e + datetime.timedelta(milliseconds=self.PERIOD_MS)
            inside = [r for r in rows if r[0] is not None and b <= r[0] <= late]
        use = inside or rows
        return {"sm_mhz": statistics.median(r[1] for r in use),
                "sm_max_mhz": max(r[2] for r in use), "reasons": sorted(reasons),
                "samples": len(use),
                "window": "timed region" if inside else "whole run (none inside the timed region)"}


# ---------------------------------------------------------------------------
# work accounting
# ---------------------------------------------------------------------------
def legal_pairs(L: int) -> int:
    return L * (L + 1) // 2


def legal_tiles(L: int, tile: int) -> int:
    nb = (L + tile - 1) // tile
    return nb * (nb + 1) // 2


def retained_pairs(kept_bits, L: int, tile: int) -> int:
    """Sum over query rows of the legal keys inside kept tiles, from the
    [.., nb, nw] keep bitmask (row = query block, bit = key block)."""
    import mass_adaptive_causal_b200 as mala
    nb = (L + tile - 1) // tile
    keep = mala.unpack_bits(kept_bits, nb)  # [..., nb, nb]
    keep = keep.reshape(-1, nb, nb).astype(np.int64)
    rows = np.minimum(L - np.arange(nb) * tile, tile)   # rows per query block
    cols = np.minimum(L - np.arange(nb) * tile, tile)   # keys per key block
    full = rows[:, None] * cols[None, :]
    diag = np.array([r * (r + 1) // 2 for r in rows])
    w = np.tril(full, -1) + np.diag(diag)
    return int((keep * w[None]).sum())


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def load_profile_traffic():
    """dram bytes per launch from the committed ncu summary, if it is current."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(path):
        try:
            return json.load(open(path))
        except Exception:
            return {}
    return {}


def reduce_max(v: float, world: int, device) -> float:
    """The largest of every rank's value (a device time: the job is as slow as
    its slowest replica); the process group's backend decides the device."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------
def count_launches(fn):
    """Kernels of this library launched by one call of ``fn``, counted from
    the CUDA activity trace (torch.profiler / CUPTI): every kernel whose name
    is in the library's namespaces."""
    import torch
    from torch.profiler import ProfilerActivity, profile
    torch.cuda.synchronize()
    try:
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            fn()
            torch.cuda.synchronize()
        names = [e.name for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA]
    except Exception:  # no activity trace (e.g. another CUPTI client such as ncu)
        return None, []
    ours = [n for n in names if any(k in n for k in ("fwd2::", "bwd100::", "bwdtest::", "dec::",
                                                          "aux::", "simt::"))]
    return len(ours), sorted(set(n.split("(")[0] for n in ours))


def run_mala(args, rank, world, local_rank):
    import torch
    import mass_adaptive_causal_b200 as mala

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    P, Dc = PREFILL, DECODE

    def to_dev(u16, shape):
        t = torch.from_numpy(u16.view(np.int16)).view(torch.bfloat16).reshape(shape)
        return t.to(dev)

    x = args._inputs
    pshape = (P.B, P.H, P.L, P.d)
    Q, K, V, dO = (to_dev(x["p" + n], pshape) for n in ("Q", "K", "V", "dO"))
    q = to_dev(x["dq"], (Dc.B, Dc.Hq, Dc.d))
    Kc = to_dev(x["dK"], (Dc.B, Dc.Hkv, Dc.Lc, Dc.d))
    Vc = to_dev(x["dV"], (Dc.B, Dc.Hkv, Dc.Lc, Dc.d))
    O = torch.empty_like(Q)
    O32 = torch.empty(Q.shape, dtype=torch.float32, device=dev)
    LSE = torch.empty((P.B, P.H, P.L), dtype=torch.float32, device=dev)
    dQ, dK, dV = torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V)
    o = torch.empty_like(q)
    ws_b = torch.empty(mala.bwd_workspace_bytes(P.B, P.H, P.L, P.d), dtype=torch.uint8, device=dev)
    ws_d = torch.empty(mala.decode_workspace_bytes(Dc.B, Dc.Hq, Dc.Hkv, Dc.Lc, Dc.d),
                       dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(tau, ev=None):
        # the training chain: only O (its float32 copy) and LSE go from the
        # forward to the backward
        if ev is not None:
            ev[0].record(stream)
        mala.mala_fwd(Q, K, V, tau=tau, out=O, lse=LSE, o32=O32)
        if ev is not None:
            ev[1].record(stream)
        mala.mala_bwd(Q, K, V, O, dO, LSE, tau=tau, workspace=ws_b, grads=(dQ, dK, dV), o32=O32)
        if ev is not None:
            ev[2].record(stream)
        mala.mala_decode(q, Kc, Vc, tau=tau, workspace=ws_d, out=o)
        if ev is not None:
            ev[3].record(stream)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    def max_over_ranks(v: float) -> float:
        return reduce_max(v, world, dev)

    def timed(tau, steps, warmup, clock=None):
        for _ in range(warmup):
            step(tau)
        mala.mala_check()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
        barrier()
        torch.cuda.synchronize()
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        if clock is not None:
            clock.mark("begin")
        start.record(stream)
        for k in range(steps):
            step(tau, evs[k])
        end.record(stream)
        torch.cuda.synchronize()
        if clock is not None:
            clock.mark("end")
        barrier()
        mala.mala_check()
        total = start.elapsed_time(end)
        fwd = [e[0].elapsed_time(e[1]) for e in evs]
        bwd = [e[1].elapsed_time(e[2]) for e in evs]
        dec = [e[2].elapsed_time(e[3]) for e in evs]
        return {"ms_per_step": max_over_ranks(total / steps),
                "fwd_ms": max_over_ranks(sum(fwd) / steps),
                "bwd_ms": max_over_ranks(sum(bwd) / steps),
                "decode_us": max_over_ranks(1000 * sum(dec) / steps)}

    # trace pass (untimed): retained work and kept decode tiles at tau=1
    def trace(tau):
        _, _, kept_f, bits_f, _ = mala.mala_fwd(Q, K, V, tau=tau, trace=True, out=O, lse=LSE,
                                                o32=O32)
        _, _, _, kept_b, bits_b = mala.mala_bwd(Q, K, V, O, dO, LSE, tau=tau, trace=True, o32=O32)
        _, kept_d, _ = mala.mala_decode(q, Kc, Vc, tau=tau, trace=True)
        mala.mala_check()
        nt = (Dc.Lc + 127) // 128
        return {"fwd_ret": retained_pairs(bits_f, P.L, P.tile),
                "bwd_ret": retained_pairs(bits_b, P.L, P.tile),
                "decode_kept_tiles": int(kept_d.sum().item()),
                "decode_tiles": Dc.B * Dc.Hkv * nt}

    clock = ClockSampler(local_rank)
    clock.start()
    t1 = timed(1.0, args.steps, args.warmup, clock=clock)
    clocks = clock.stop()
    work1 = trace(1.0)
    launches, kernels = count_launches(lambda: step(1.0))
    work1["launches_per_step"] = launches
    work1["kernels"] = kernels
    dense = timed(0.0, max(1, min(args.steps, 3)), 1) if not args.no_dense else None
    e2e = None if args.no_e2e else run_e2e(args, x, dev, world, max_over_ranks)
    del Q, K, V, dO, q, Kc, Vc, O, O32, LSE, dQ, dK, dV, o, ws_b, ws_d
    torch.cuda.empty_cache()
    return t1, work1, dense, clocks, e2e


def run_e2e(args, x, dev, world, max_over_ranks):
    """Same metric through the public API with inputs in pinned HOST memory:
    each step copies the inputs host->device, runs the three calls and copies
    the results back (O, LSE, dQ, dK, dV and the decode output). The decode
    cache's copy runs on a second stream beside the prefill's work."""
    import torch
    import mass_adaptive_causal_b200 as mala
    P, Dc = PREFILL, DECODE

    def pinned(u16, shape):
        return torch.from_numpy(u16.view(np.int16)).view(torch.bfloat16).reshape(shape).pin_memory()

    pshape = (P.B, P.H, P.L, P.d)
    hQ, hK, hV, hdO = (pinned(x["p" + n], pshape) for n in ("Q", "K", "V", "dO"))
    hq = pinned(x["dq"], (Dc.B, Dc.Hq, Dc.d))
    hKc = pinned(x["dK"], (Dc.B, Dc.Hkv, Dc.Lc, Dc.d))
    hVc = pinned(x["dV"], (Dc.B, Dc.Hkv, Dc.Lc, Dc.d))
    outs_h = {n: torch.empty(pshape, dtype=torch.bfloat16).pin_memory() for n in ("O", "dQ", "dK", "dV")}
    lse_h = torch.empty((P.B, P.H, P.L), dtype=torch.float32).pin_memory()
    o_h = torch.empty((Dc.B, Dc.Hq, Dc.d), dtype=torch.bfloat16).pin_memory()
    dQ_ = {n: torch.empty(pshape, dtype=torch.bfloat16, device=dev) for n in ("Q", "K", "V", "dO")}
    q_, Kc_, Vc_ = (torch.empty(t.shape, dtype=t.dtype, device=dev) for t in (hq, hKc, hVc))
    h2d = sum(t.numel() * t.element_size() for t in (hQ, hK, hV, hdO, hq, hKc, hVc))
    d2h = sum(t.numel() * t.element_size() for t in outs_h.values()) + lse_h.numel() * 4 + \
        o_h.numel() * 2

    # The decode step's inputs (the 8.6 GB cache) go over a second stream, so
    # their copy overlaps the prefill's compute and its results' copy back;
    # that stream first waits for the main one (the prefill's inputs go first,
    # and the previous step's decode has read the cache before it is refilled)
    main = torch.cuda.current_stream(dev)
    side = torch.cuda.Stream(device=dev)

    def step():
        for n, h in zip(("Q", "K", "V", "dO"), (hQ, hK, hV, hdO)):
            dQ_[n].copy_(h, non_blocking=True)
        side.wait_stream(main)
        with torch.cuda.stream(side):
            q_.copy_(hq, non_blocking=True)
            Kc_.copy_(hKc, non_blocking=True)
            Vc_.copy_(hVc, non_blocking=True)
        O, LSE, O32 = mala.mala_fwd(dQ_["Q"], dQ_["K"], dQ_["V"], tau=1.0, o32=True)
        dQ, dK, dV = mala.mala_bwd(dQ_["Q"], dQ_["K"], dQ_["V"], O, dQ_["dO"], LSE, tau=1.0,
                                   o32=O32)
        for n, t in (("O", O), ("dQ", dQ), ("dK", dK), ("dV", dV)):
            outs_h[n].copy_(t, non_blocking=True)
        lse_h.copy_(LSE, non_blocking=True)
        main.wait_stream(side)
        o = mala.mala_decode(q_, Kc_, Vc_, tau=1.0)
        o_h.copy_(o, non_blocking=True)

    steps = max(1, min(args.steps, 3))
    for _ in range(max(1, min(args.warmup, 2))):
        step()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        step()
    e.record()
    torch.cuda.synchronize()
    mala.mala_check()
    ms = max_over_ranks(s.elapsed_time(e) / steps)
    return {"value": ms, "unit": "ms", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "steps": steps}


# ---------------------------------------------------------------------------
# the CPU oracle (reported baseline; also the --impl reference arm)
# ---------------------------------------------------------------------------
def oracle_sample(x, budget_s: float):
    """Time the CPU oracle on a bounded sample of the same workload and
    extrapolate to milliseconds per step. Returns (ms_per_step, cores, desc)."""
    import oracle
    cores = oracle.threads(len(os.sched_getaffinity(0)))
    P, Dc = PREFILL, DECODE
    T = P.tile
    nb = P.L // T

    def f64(u16, shape):
        return (u16.astype(np.uint32) << 16).view(np.float32).astype(np.float64).reshape(shape)

    h = 0
    Qh = f64(x["pQ"][h], (P.L, P.d))
    Kh = f64(x["pK"][h], (P.L, P.d))
    Vh = f64(x["pV"][h], (P.L, P.d))
    dOh = f64(x["pdO"][h], (P.L, P.d))
    # forward: the last `nq` query blocks (each visits every key tile)
    nq = max(1, cores)
    t0 = time.perf_counter()
    fr = oracle.fwd(Qh, Kh, Vh, tile=T, tau=1.0, qblocks=(nb - nq, nb))
    t_fwd = time.perf_counter() - t0
    tiles_fwd = sum(i + 1 for i in range(nb - nq, nb))
    fwd_per_tile = t_fwd / tiles_fwd
    # backward: dK/dV of the last `nk` key blocks and dQ of the last block
    nk = max(1, cores)
    LSE = np.nan_to_num(fr["LSE"])
    Oh = np.nan_to_num(fr["O"])
    t0 = time.perf_counter()
    oracle.bwd(Qh, Kh, Vh, Oh, dOh, LSE, tile=T, tau=1.0, qblocks=[nb - 1],
               kblocks=list(range(nb - nk, nb)))
    t_bwd = time.perf_counter() - t0
    tiles_bwd = nb + sum(nb - j for j in range(nb - nk, nb))
    bwd_per_tile = t_bwd / tiles_bwd
    # decode: one group
    nt = Dc.Lc // 128
    G = Dc.Hq // Dc.Hkv
    q0 = f64(x["dq"][0], (G, Dc.d))
    K0 = f64(x["dK"][0], (1, Dc.Lc, Dc.d))
    V0 = f64(x["dV"][0], (1, Dc.Lc, Dc.d))
    t0 = time.perf_counter()
    oracle.decode(q0, K0, V0, tau=1.0)
    t_dec = time.perf_counter() - t0
    total_tiles = P.B * P.H * nb * (nb + 1) // 2
    ms = 1000 * (fwd_per_tile * total_tiles + bwd_per_tile * total_tiles +
                 t_dec * Dc.B * Dc.Hkv)
    desc = (f"fwd: last {nq} query blocks of head 0 ({tiles_fwd} tiles, {t_fwd:.1f}s); "
            f"bwd: dK/dV of last {nk} key blocks + dQ of last query block ({tiles_bwd} tiles, "
            f"{t_bwd:.1f}s); decode: 1 of {Dc.B * Dc.Hkv} groups ({t_dec:.1f}s); extrapolated "
            f"per tile pair / per group to the full step")
    return ms, cores, desc


# ---------------------------------------------------------------------------
def profile_case(args):
    """A small case of one call for ncu: long_128k recipe at length --L
    (B=1, H=8; Q/K/V larger than L2 from L=32768), or a decode step with
    B=4 over a 131072-key cache. Runs `--warmup` untimed launches then
    `--launches` more and prints their mean time."""
    import torch
    import mass_adaptive_causal_b200 as mala
    torch.cuda.set_device(0)
    if args.profile in ("fwd", "bwd"):
        x = synth.prefill_inputs(PREFILL, L=args.L)
        t = {n: torch.tensor(x[n]).to(torch.bfloat16).cuda() for n in ("Q", "K", "V", "dO")}
        tau = args.tau
        O, LSE, O32 = mala.mala_fwd(t["Q"], t["K"], t["V"], tau=tau, o32=True)
        run = (lambda: mala.mala_fwd(t["Q"], t["K"], t["V"], tau=tau, out=O, lse=LSE, o32=O32)) \
            if args.profile == "fwd" else \
            (lambda: mala.mala_bwd(t["Q"], t["K"], t["V"], O, t["dO"], LSE, tau=tau, o32=O32))
    else:
        cfg = synth.DecodeConfig("profile", 4, 4, DECODE.Hq, DECODE.Hkv, DECODE.Lc, DECODE.d,
                                 128, DECODE.rho, DECODE.n_pairs, DECODE.n_query_targets)
        x = synth.decode_inputs(cfg)
        q, Kc, Vc = (torch.tensor(x[n]).to(torch.bfloat16).cuda() for n in ("q", "K", "V"))
        run = lambda: mala.mala_decode(q, Kc, Vc, tau=1.0)
    for _ in range(args.warmup):
        run()
    mala.mala_check()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(args.launches):
        run()
    e.record()
    torch.cuda.synchronize()
    mala.mala_check()
    print(json.dumps({"profile": args.profile, "L": args.L, "tau": args.tau,
                      "ms_per_launch": s.elapsed_time(e) / args.launches}), flush=True)


def tau_study(args):
    """Slots per query, omitted mass and output error against dense attention
    over a sweep of tau, on the long_128k prefill and the decode_128k step
    (group rows and per-head rows). The omitted mass of row r is
    1 - exp(LSE_tau - LSE_dense): LSE_tau normalizes over the kept keys only.
    Everything runs on the GPU kernels; one JSON line."""
    import torch
    import mass_adaptive_causal_b200 as mala
    torch.cuda.set_device(0)
    P, Dc = PREFILL, DECODE
    x = generate_inputs(args.workers or min(16, os.cpu_count() or 1))

    def to_dev(u16, shape):
        return torch.from_numpy(u16.view(np.int16)).view(torch.bfloat16).reshape(shape).cuda()

    pshape = (P.B, P.H, P.L, P.d)
    Q, K, V = (to_dev(x["p" + n], pshape) for n in ("Q", "K", "V"))
    O0, L0 = mala.mala_fwd(Q, K, V, tau=0.0)

    def timed(fn, reps=3):
        fn()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(reps):
            fn()
        e.record()
        torch.cuda.synchronize()
        return s.elapsed_time(e) / reps

    rows = []
    for tau in (0.0625, 0.25, 1.0, 4.0, 16.0):
        O, LSE, kept, bits = mala.mala_fwd(Q, K, V, tau=tau, trace=True)
        mala.mala_check()
        om = (1.0 - torch.exp(LSE.double() - L0.double())).clamp_min(0.0)
        rel = float(torch.linalg.norm((O.float() - O0.float()).flatten()) /
                    torch.linalg.norm(O0.float().flatten()))
        rows.append({"tau": tau, "fwd_ms": timed(lambda: mala.mala_fwd(Q, K, V, tau=tau)),
                     "slots_per_query": retained_pairs(bits, P.L, P.tile) / (P.B * P.H * P.L),
                     "omitted_mass_mean": float(om.mean()), "omitted_mass_max": float(om.max()),
                     "bound_tau_over_1_plus_tau": tau / (1 + tau), "out_rel_l2_vs_dense": rel})
    del Q, K, V, O0, L0
    q = to_dev(x["dq"], (Dc.B, Dc.Hq, Dc.d))
    Kc = to_dev(x["dK"], (Dc.B, Dc.Hkv, Dc.Lc, Dc.d))
    Vc = to_dev(x["dV"], (Dc.B, Dc.Hkv, Dc.Lc, Dc.d))
    o0 = mala.mala_decode(q, Kc, Vc, tau=0.0)
    nt = (Dc.Lc + 127) // 128
    drows = []
    for per_head in (False, True):
        for tau in (0.25, 1.0, 4.0):
            o, kept, _ = mala.mala_decode(q, Kc, Vc, tau=tau, trace=True, per_head=per_head)
            mala.mala_check()
            units = Dc.Hq if per_head else Dc.Hkv
            rel = float(torch.linalg.norm((o.float() - o0.float()).flatten()) /
                        torch.linalg.norm(o0.float().flatten()))
            drows.append({"rows": "per_head" if per_head else "group", "tau": tau,
                          "decode_us": 1000 * timed(lambda: mala.mala_decode(
                              q, Kc, Vc, tau=tau, per_head=per_head)),
                          "kept_tile_frac": float(kept.sum()) / (Dc.B * units * nt),
                          "out_rel_l2_vs_dense": rel})
    print(json.dumps({"study": "tau_sweep", "prefill": {"workload": "long_128k", "rows": rows},
                      "decode": {"workload": "decode_128k", "rows": drows}}), flush=True)


# ---------------------------------------------------------------------------
# matched-work policy study (matched_8k): at the per-block tile budget of the
# rule's own GPU keep set, other allocations of the same number of tiles are
# compared by the dense probability mass they leave out and by their output
# error against dense attention (MassAlloc Attention; jaehun.me review,
# "Matched-work study", Table 1; agihunt.info summary, matched-work paragraph)
# ---------------------------------------------------------------------------
# calibration draws of the head-position policy: sequence indices
# CAL_SEQ0 + H k + h of the same config (independent streams, never a
# benchmarked sequence)
CAL_SEQ0 = 500
N_CAL = 2
POLICIES = ("mala", "position_static", "head_position_static", "per_instance_oracle")


def bf16_round(a):
    """float64 -> nearest bfloat16 -> float64 (the inputs the kernels see)."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).double().numpy()


def dense_row_tile_mass(Q, K, tile, scale):
    """Host float64 analysis: dense causal softmax probabilities P (L, L) of
    one slice and, per row r and key tile j, the probability row r puts on
    tile j's keys (L, nb)."""
    L = Q.shape[0]
    S = (Q @ K.T) * scale
    S[np.arange(L)[None, :] > np.arange(L)[:, None]] = -np.inf
    S -= S.max(axis=1, keepdims=True)
    P = np.exp(S)
    P /= P.sum(axis=1, keepdims=True)
    nb = (L + tile - 1) // tile
    Pp = np.zeros((L, nb * tile))
    Pp[:, :L] = P
    return P, Pp.reshape(L, nb, tile).sum(axis=2)


def block_mass(row_mass, tile):
    """(L, nb) per-row tile mass -> (nb, nb) summed over each query block."""
    L, nb = row_mass.shape
    pad = np.zeros((nb * tile, nb))
    pad[:L] = row_mass
    return pad.reshape(nb, tile, nb).sum(axis=1)


def position_static_keep(counts):
    """Per query block i: the diagonal tile, the first (sink) tile, then the
    nearest earlier tiles, counts[i] of them; the same for every input."""
    nb = len(counts)
    keep = np.zeros((nb, nb), np.uint8)
    for i in range(nb):
        order = [i] + ([0] if i > 0 else []) + list(range(i - 1, 0, -1))
        keep[i, order[:counts[i]]] = 1
    return keep


def top_keep(score, counts):
    """Per query block i: the counts[i] legal tiles of largest score."""
    nb = len(counts)
    keep = np.zeros((nb, nb), np.uint8)
    for i in range(nb):
        order = np.argsort(-score[i, :i + 1], kind="stable")
        keep[i, order[:counts[i]]] = 1
    return keep


def restricted_output(P, V, keep, tile):
    """Softmax restricted to the kept tiles, times V, and the per-row mass
    left out."""
    L = P.shape[0]
    blk = np.arange(L) // tile
    Pk = np.where(keep[blk][:, blk].astype(bool), P, 0.0)
    kept = Pk.sum(axis=1)
    return (Pk @ V) / kept[:, None], 1.0 - kept


def policy_study(args):
    """One JSON line: per allocation policy, the mean omitted mass and the
    output rel-L2 against dense attention, on matched_8k (8 heads, L=8192),
    each policy given the rule's per-block tile counts from mala_fwd's keep
    bits. Dense probabilities are host float64 analysis of the bf16 inputs."""
    import torch
    import mass_adaptive_causal_b200 as mala
    torch.cuda.set_device(0)
    cfg = synth.CONFIGS["matched_8k"]
    L, H, d, tile = cfg.L, cfg.H, cfg.d, cfg.tile
    scale = 1.0 / np.sqrt(d)
    x = synth.prefill_inputs(cfg, with_grad=False)
    host = {n: bf16_round(x[n]) for n in ("Q", "K", "V")}
    dev = {n: torch.from_numpy(host[n]).to(torch.bfloat16).cuda() for n in host}
    O, LSE, kept, bits = mala.mala_fwd(dev["Q"], dev["K"], dev["V"], tau=1.0, trace=True)
    mala.mala_check()
    nb = (L + tile - 1) // tile
    keep_gpu = mala.unpack_bits(bits, nb)
    O_gpu = O.float().cpu().numpy()
    u = synth.unit_vector(cfg.config_seed, d)
    acc = {n: {"omitted_mass_mean": 0.0, "out_rel_l2": 0.0} for n in POLICIES}
    kernel_err = 0.0
    t0 = time.time()
    for h in range(H):
        Q, K, V = host["Q"][0, h], host["K"][0, h], host["V"][0, h]
        P, rm = dense_row_tile_mass(Q, K, tile, scale)
        cal = np.zeros((nb, nb))
        for k in range(N_CAL):
            sq = synth.prefill_sequence(cfg.config_seed, CAL_SEQ0 + H * k + h, L, d, cfg.rho,
                                        cfg.n_pairs, u, with_grad=False)
            _, rmc = dense_row_tile_mass(bf16_round(sq["Q"]), bf16_round(sq["K"]), tile, scale)
            cal += block_mass(rmc, tile)
        kg = keep_gpu[0, h]
        counts = kg.sum(axis=1)
        keeps = {"mala": kg, "position_static": position_static_keep(counts),
                 "head_position_static": top_keep(cal, counts),
                 "per_instance_oracle": top_keep(block_mass(rm, tile), counts)}
        O_dense = P @ V
        nrm = np.linalg.norm(O_dense)
        for name, kp in keeps.items():
            assert np.array_equal(kp.sum(axis=1), counts)
            Oz, om = restricted_output(P, V, kp, tile)
            acc[name]["omitted_mass_mean"] += om.mean() / H
            acc[name]["out_rel_l2"] += np.linalg.norm(Oz - O_dense) / nrm / H
        kernel_err += np.linalg.norm(O_gpu[0, h] - O_dense) / nrm / H
    print(json.dumps({"study": "matched_work", "workload": "matched_8k", "heads": H, "L": L,
                      "slots_per_query": retained_pairs(bits, L, tile) / (H * L),
                      "policies": acc, "mala_kernel_out_rel_l2": kernel_err,
                      "calibration_draws": N_CAL, "host_seconds": time.time() - t0}), flush=True)


# ---------------------------------------------------------------------------
# per-workload report: configurations 0-2 (the tiny float32 case, the
# matched-work shape and the length sweep), each at tau=1 and tau=0
# ---------------------------------------------------------------------------
PER_WORKLOAD = ["tiny_f32", "matched_8k"] + [f"sweep_L{L}" for L in (1024, 2048, 4096, 8192, 16384,
                                                                       32768)]
# heads whose keep sets the oracle recomputes (near-threshold flip counts and
# the oracle's own time on this workload); "fwd" = forward only
ORACLE_HEADS = {"tiny_f32": (1, "both"), "matched_8k": (8, "both"), "sweep_L1024": (16, "both"),
                "sweep_L2048": (16, "both"), "sweep_L4096": (16, "both"),
                "sweep_L8192": (4, "both"), "sweep_L16384": (1, "both"),
                "sweep_L32768": (1, "fwd")}
FP32_SIMT_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12  # 148 SMs x 128 FP32 FMA/clk at 1965 MHz


def workload_oracle(cfg, host, gbits_f, gbits_b, n_heads, which, tau=1.0):
    """The CPU oracle on ``n_heads`` heads of this workload (the values the GPU
    sees, rounded on the host): its wall time on this host's cores, and the
    GPU keep sets compared with its own -- mismatches inside the
    near-threshold band are counted (both decisions are correct there), any
    other mismatch is counted separately (it must be 0)."""
    import mass_adaptive_causal_b200 as mala
    import oracle
    sys.path.insert(0, ROOT)
    from tests.parity import NEAR
    cores = oracle.threads(len(os.sched_getaffinity(0)))
    nb = (cfg.L + cfg.tile - 1) // cfg.tile
    tril = np.tril(np.ones((nb, nb), bool))
    flips_f = flips_b = other = 0
    t_cpu = 0.0
    for h in range(n_heads):
        Qd, Kd, Vd, dOd = (host[n][0, h] for n in ("Q", "K", "V", "dO"))
        t0 = time.perf_counter()
        ref = oracle.fwd(Qd, Kd, Vd, tile=cfg.tile, tau=tau, want_margin=True)
        g = None
        if which == "both":
            g = oracle.bwd(Qd, Kd, Vd, ref["O"], dOd, ref["LSE"], tile=cfg.tile, tau=tau,
                           want_margin=True)
        t_cpu += time.perf_counter() - t0
        gk = mala.unpack_bits(gbits_f[0, h], nb)
        bad = set()
        for i in range(nb):
            for j in range(i, -1, -1):
                if gk[i, j] != ref["keep"][i, j]:
                    if abs(ref["margin"][i, j]) <= NEAR:
                        flips_f += 1
                    else:
                        other += 1
                    bad.add(i)
                    break  # later tiles of this block follow a different state
        if g is not None:
            gb = mala.unpack_bits(gbits_b[0, h], nb)
            diff = (gb.astype(bool) != g["keep"].astype(bool)) & tril
            for i, j in zip(*np.nonzero(diff)):
                if i in bad:
                    continue
                if abs(g["margin"][i, j]) <= NEAR:
                    flips_b += 1
                else:
                    other += 1
    per_head = t_cpu / max(1, n_heads)
    return {"heads": n_heads, "passes": "fwd+bwd" if which == "both" else "fwd", "cpu_s": t_cpu,
            "cores": cores, "cpu_s_all_heads_extrapolated": per_head * cfg.B * cfg.H,
            "near_threshold_flips_fwd": flips_f, "near_threshold_flips_bwd": flips_b,
            "mismatches_outside_band": other}


def per_workload(dev, peaks, oracle_leg=True, reps=5):
    """Configurations 0-2 on the GPU kernels, each at tau=1 and at tau=0
    (the in-house dense comparison): ms, effective TFLOP/s and fraction of
    the roofline, retained slots per query, omitted mass and O/dQ/dK/dV error
    against tau=0, and (oracle_leg) the oracle's time and the near-threshold
    flip counts on sampled heads."""
    import torch
    import mass_adaptive_causal_b200 as mala
    out = []
    for name in PER_WORKLOAD:
        cfg = synth.CONFIGS[name]
        x = synth.prefill_inputs(cfg)
        dt = torch.float32 if cfg.dtype == "f32" else torch.bfloat16
        host = {n: torch.tensor(x[n]).to(dt) for n in ("Q", "K", "V", "dO")}
        t = {n: v.to(dev) for n, v in host.items()}
        res = {"workload": name, "shape": f"B{cfg.B} H{cfg.H} L{cfg.L} d{cfg.d} tile{cfg.tile}",
               "dtype": "f32" if cfg.dtype == "f32" else "bf16"}
        d, L = cfg.d, cfg.L
        P_legal = cfg.B * cfg.H * legal_pairs(L)
        runs = {}
        for tau in (1.0, 0.0):
            o32 = dt == torch.bfloat16
            O, LSE, kept, bits, *r = mala.mala_fwd(t["Q"], t["K"], t["V"], tau=tau, trace=True,
                                                   o32=o32)
            O32 = r[0] if o32 else O
            dQ, dK, dV, kept_b, bits_b = mala.mala_bwd(t["Q"], t["K"], t["V"], O, t["dO"], LSE,
                                                       tau=tau, trace=True,
                                                       o32=O32 if o32 else None)
            mala.mala_check()

            def ev_time(fn):
                fn()
                ts = []
                for _ in range(reps):
                    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    s.record()
                    fn()
                    e.record()
                    torch.cuda.synchronize()
                    ts.append(s.elapsed_time(e))
                return statistics.median(ts)
            f_ms = ev_time(lambda: mala.mala_fwd(t["Q"], t["K"], t["V"], tau=tau, out=O, lse=LSE,
                                                 o32=O32 if o32 else None))
            b_ms = ev_time(lambda: mala.mala_bwd(t["Q"], t["K"], t["V"], O, t["dO"], LSE, tau=tau,
                                                 o32=O32 if o32 else None))
            fret = retained_pairs(bits, L, cfg.tile)
            bret = retained_pairs(bits_b, L, cfg.tile)
            f_fl = 2 * d * P_legal + 2 * d * fret
            b_fl = 2 * d * P_legal + 8 * d * bret
            peak = FP32_SIMT_TFLOPS if cfg.dtype == "f32" else peaks["bf16_tflops"]
            f_tf, b_tf = f_fl / (f_ms * 1e-3) / 1e12, b_fl / (b_ms * 1e-3) / 1e12
            runs[tau] = {"O": O32.float(), "LSE": LSE.double(), "dQ": dQ.float(), "dK": dK.float(),
                         "dV": dV.float(), "bits": bits, "bits_b": bits_b}
            res[f"tau{int(tau)}"] = {
                "fwd_ms": f_ms, "bwd_ms": b_ms, "fwd_tflops_eff": f_tf, "bwd_tflops_eff": b_tf,
                "fwd_frac": f_tf / peak, "bwd_frac": b_tf / peak,
                "peak": "fp32 SIMT nominal" if cfg.dtype == "f32" else "bf16 burst (measured)",
                "fwd_slots_per_query": fret / (cfg.B * cfg.H * L),
                "bwd_slots_per_query": bret / (cfg.B * cfg.H * L)}
        a, z = runs[1.0], runs[0.0]
        om = (1.0 - torch.exp(a["LSE"] - z["LSE"])).clamp_min(0.0).flatten()

        def rel(n):
            return float(torch.linalg.norm((a[n] - z[n]).flatten()) /
                         torch.linalg.norm(z[n].flatten()))
        res["tau1_vs_tau0"] = {"omitted_mass_mean": float(om.mean()),
                               "omitted_mass_p95": float(torch.quantile(om.float(), 0.95))
                               if om.numel() <= 1 << 24 else None,
                               "omitted_mass_max": float(om.max()), "O_rel_l2": rel("O"),
                               "dQ_rel_l2": rel("dQ"), "dK_rel_l2": rel("dK"), "dV_rel_l2": rel("dV"),
                               "fwd_speedup": res["tau0"]["fwd_ms"] / res["tau1"]["fwd_ms"],
                               "bwd_speedup": res["tau0"]["bwd_ms"] / res["tau1"]["bwd_ms"]}
        if oracle_leg:
            nh, which = ORACLE_HEADS[name]
            hostd = {n: v.double().numpy() for n, v in host.items()}
            res["oracle"] = workload_oracle(cfg, hostd, a["bits"], a["bits_b"], nh, which)
        out.append(res)
        del t, runs, a, z
        torch.cuda.empty_cache()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="mala", choices=["mala", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workers", type=int, default=0)
    ap.add_argument("--profile", choices=["fwd", "bwd", "decode"], default=None,
                    help="run only a small case of one call (for ncu captures)")
    ap.add_argument("--L", type=int, default=32768, help="sequence length of --profile")
    ap.add_argument("--launches", type=int, default=2, help="timed launches of --profile")
    ap.add_argument("--tau", type=float, default=1.0, help="tau of --profile")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="skip the per-workload report of configurations 0-2")
    ap.add_argument("--study", choices=["tau", "policy"], default=None,
                    help="tau: sweep of tau (slots, omitted mass, error against dense); policy: "
                         "matched-work allocation policies on matched_8k; one JSON line each")
    args = ap.parse_args()
    if args.profile:
        return profile_case(args)
    if args.study == "tau":
        return tau_study(args)
    if args.study == "policy":
        return policy_study(args)
    args.warmup = max(3, args.warmup)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    ncpu = len(os.sched_getaffinity(0))
    workers = args.workers or max(1, min(32, ncpu // max(1, world)))

    if args.impl == "reference":
        if rank != 0:
            return
        x = generate_inputs(workers)
        per_step = []
        cores, desc = None, ""
        for _ in range(args.warmup + args.steps):
            ms, cores, desc = oracle_sample(x, 30.0)
            per_step.append(ms)
        ms = statistics.mean(per_step[args.warmup:])
        line = {"impl": "reference", "metric": "ms per step (fwd+bwd at 128K + one decode step at 128K)",
                "value": ms, "unit": "ms", "n_gpus": args.gpus, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": False,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": WORKLOAD},
                "cpu_baseline": {"value": ms, "unit": "ms", "cores": cores, "kind": "oracle",
                                 "sample": desc},
                "e2e": {"value": ms, "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    # generate inputs before any CUDA call (spawn pool)
    x = generate_inputs(workers, seed_shift=0 if world == 1 else 100 * rank)
    args._inputs = x
    if world > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    t1, work, dense, clocks, e2e = run_mala(args, rank, world, local_rank)

    P, Dc = PREFILL, DECODE
    peaks = load_peaks()
    d = P.d
    P_legal = P.B * P.H * legal_pairs(P.L)
    # effective work: every legal QK plus the retained post-score work
    # (forward P.V: 2d per retained pair; backward P, dV, dP, dK, dQ: 8d)
    fwd_flop = 2 * d * P_legal + 2 * d * work["fwd_ret"]
    bwd_flop = 2 * d * P_legal + 8 * d * work["bwd_ret"]
    fwd_tf = fwd_flop / (t1["fwd_ms"] * 1e-3) / 1e12
    bwd_tf = bwd_flop / (t1["bwd_ms"] * 1e-3) / 1e12
    kc_bytes = Dc.B * Dc.Hkv * Dc.Lc * Dc.d * 2
    nt = Dc.Lc // 128
    tile_bytes = 128 * Dc.d * 2
    dec_bytes = kc_bytes + 2 * work["decode_kept_tiles"] * tile_bytes + \
        Dc.B * Dc.Hq * (2 * Dc.d * 2 + nt * 8 * 2)
    dec_gbs = dec_bytes / (t1["decode_us"] * 1e-6) / 1e9
    traffic = load_profile_traffic()
    sus = peaks["bf16_tflops_sustained"] or peaks["bf16_tflops"]
    src = peaks["source"] + " (burst bf16 cuBLAS)"
    # the forward is one kernel per call, so its CUDA-event bracket is that
    # kernel's launch time; the backward call is four kernels, the
    # recomputing skip test among them, and its bracket covers them all
    roof = {"bound": "tensor", "kernel": "mala::fwd2::fwd_pair_kernel", "achieved": fwd_tf,
            "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": fwd_tf / peaks["bf16_tflops"],
            "traffic": traffic.get("fwd_pair_kernel"), "peak_source": src,
            "frac_of_sustained": fwd_tf / sus}
    roof_bwd = {"bound": "tensor", "call": "mala_bwd (row terms, skip test, work pass, dQ convert)",
                "achieved": bwd_tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": bwd_tf / peaks["bf16_tflops"], "traffic": traffic.get("bwd_call"),
                "peak_source": src, "frac_of_sustained": bwd_tf / sus}
    roof_dec = {"bound": "hbm", "call": "mala_decode", "achieved": dec_gbs, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": dec_gbs / peaks["hbm_gbs"],
                "traffic": traffic.get("decode_call")}

    line = {
        "metric": "ms per step (fwd+bwd at 128K + one decode step at 128K)",
        "value": t1["ms_per_step"], "unit": "ms", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t1["ms_per_step"], "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "tau": 1.0, "l2": "inputs larger than L2 (no flush)",
                   "parallelism": f"replicas x{world} (independent heads/sequences per rank)"},
        "fwd_ms": t1["fwd_ms"], "bwd_ms": t1["bwd_ms"], "decode_us": t1["decode_us"],
        "fwd_tflops_eff": fwd_tf, "bwd_tflops_eff": bwd_tf,
        "fwd_frac_bf16": fwd_tf / peaks["bf16_tflops"], "bwd_frac_bf16": bwd_tf / peaks["bf16_tflops"],
        "decode_gbs": dec_gbs, "decode_frac_hbm": dec_gbs / peaks["hbm_gbs"],
        "decode_bytes": dec_bytes,
        "fwd_slots_per_query": work["fwd_ret"] / (P.B * P.H * P.L),
        "bwd_slots_per_query": work["bwd_ret"] / (P.B * P.H * P.L),
        "decode_kept_tile_frac": work["decode_kept_tiles"] / work["decode_tiles"],
        "roofline": roof, "roofline_bwd": roof_bwd, "roofline_decode": roof_dec,
        "clocks": clocks,
        "gpu_launches": (args.steps * work["launches_per_step"]
                         if work["launches_per_step"] is not None else None),
        "gpu_launches_per_step": work["launches_per_step"], "kernels": work["kernels"],
    }
    if dense is not None:
        line["dense_tau0"] = {"fwd_ms": dense["fwd_ms"], "bwd_ms": dense["bwd_ms"],
                              "decode_us": dense["decode_us"],
                              "fwd_speedup": dense["fwd_ms"] / t1["fwd_ms"],
                              "bwd_speedup": dense["bwd_ms"] / t1["bwd_ms"],
                              "decode_speedup": dense["decode_us"] / t1["decode_us"],
                              "fwd_tflops": 4 * d * P_legal / (dense["fwd_ms"] * 1e-3) / 1e12,
                              "bwd_tflops": 10 * d * P_legal / (dense["bwd_ms"] * 1e-3) / 1e12}
        for k in ("fwd", "bwd"):
            line["dense_tau0"][k + "_frac_bf16"] = line["dense_tau0"][k + "_tflops"] / peaks["bf16_tflops"]
    if e2e is not None:
        line["e2e"] = e2e
    if rank == 0 and world == 1 and not args.no_per_workload:
        import torch
        line["per_workload"] = per_workload(torch.device("cuda", local_rank), peaks,
                                            oracle_leg=not args.no_cpu_baseline)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        ms, cores, desc = oracle_sample(x, 30.0)
        line["cpu_baseline"] = {"value": ms, "unit": "ms", "cores": cores, "kind": "oracle",
                                "sample": desc}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
