#!/usr/bin/env python3
"""MSA hot-path benchmark on B200: prefill tokens/s and decode tokens/s.

One step = one msa_prefill over the prefill workload (index branch, query
lists, Main Branch, merge; by default the 1M-token workload, its query axis
processed in chunks that fit a 96 GiB workspace) plus one msa_decode step over
the decode workload (16 sequences of 256K cached tokens and one of 1M).  The
32K and 128K prefill workloads are then measured the same way, prefill only,
and reported under "extra".  Inputs are seeded synthetic tensors (``synth``)
resident in HBM; each is larger than the 126 MB L2 (Q is 512 MiB at 32K and
16 GiB at 1M, the decode caches 21 GiB), so no flush is needed between steps.
Kernel times come from CUDA events that the library records on its own
stream at kernel boundaries (msa_set_phase_events).

Prints exactly one JSON line on rank 0.  ``--impl reference`` times the fp64
CPU oracle on bounded samples of the same workload instead.
Launch with torchrun for N > 1 GPUs: every rank runs an independent replica
(the path has no exchange step), ``value`` sums all ranks' tokens over the
slowest rank's time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "MSA prefill tokens/s & decode tokens/s on 1 B200; % of tensor/HBM roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# B200 datasheet figures, reported beside the measured fractions (the targets
# are judged on the measured peaks)
NOMINAL_PEAKS = {"hbm_gbs": 7700.0, "bf16_tflops": 2250.0}
DEFAULT_WORKLOAD = "prefill_1m"
DEFAULT_EXTRA = "prefill_32k,prefill_128k"
PREFILL_PHASES = ("index_select", "block_query_lists", "main_branch", "merge")
DECODE_PHASES = ("decode_index", "decode_select_attend")


# --------------------------------------------------------------------------
# algorithmic work (what each kernel must at least do, independent of design)
# --------------------------------------------------------------------------

def index_flops(N: int, G: int, d_idx: int, block: int = 128) -> float:
    """2 * d_idx * G * sum_t (keys of the non-local visible blocks of t)."""
    t = np.arange(N, dtype=np.int64)
    return 2.0 * d_idx * G * float(((t // block) * block).sum())


def dense_flops(N: int, H: int, d: int) -> float:
    """Dense causal attention over the same heads: 4 * d * H * N(N+1)/2."""
    return 4.0 * d * H * N * (N + 1) / 2.0


def msa_model_flops(N: int, H: int, G: int, d: int, d_idx: int, top_k: int = 16,
                    block: int = 128) -> float:
    """Index scoring over every visible token plus the Main Branch budget, per
    the pages' O(N) dense vs O(k B_k) description (no kernel detail)."""
    t = np.arange(N, dtype=np.float64)
    idx = 2.0 * d_idx * G * (t + 1).sum()
    main = 4.0 * d * H * np.minimum(t + 1, top_k * block).sum()
    return float(idx + main)


def prefill_work(ids: np.ndarray, H: int, d: int, block: int = 128) -> dict:
    """Exact Main Branch work of one selection ids [N, G, k]."""
    N, G, k = ids.shape
    HG = H // G
    t = np.arange(N, dtype=np.int64)[:, None, None]
    valid = ids >= 0
    keys = np.where(valid, np.minimum(block, t - ids.astype(np.int64) * block + 1), 0)
    slots = int(valid.sum())
    pairs = slots * HG
    main_flops = 4.0 * d * HG * float(keys.sum())
    # gathered q row (2d) + partial o (2d fp16) + its (m, l) (8) per (token, head, block)
    main_bytes = pairs * (2 * d + 2 * d + 8.0)
    merge_bytes = pairs * (2 * d + 8.0) + N * H * 2.0 * d + N * G * k * 4.0
    csr_bytes = 3.0 * N * G * k * 4.0
    return dict(slots=slots, pairs=pairs, main_flops=main_flops, main_bytes=main_bytes,
                merge_bytes=merge_bytes, csr_bytes=csr_bytes,
                selected_keys=float(keys.sum()) / max(1, N * G))


def decode_work(seq_lens, H: int, G: int, d: int, d_idx: int, ids: np.ndarray,
                block: int = 128, fp8_index: bool = False) -> dict:
    """Bytes and FLOPs of one decode step.  The index scan reads every non-local
    cached key once (bf16: 2 bytes a value; e4m3: 1 byte a value plus its row's
    4-byte scale) and each sequence's G index queries; the attention reads the
    K and V rows of the selected blocks."""
    lens = np.asarray(seq_lens, dtype=np.int64)
    nb = (lens + block - 1) // block
    scan_keys = float(((nb - 1) * block).sum())
    if fp8_index:
        idx_bytes = scan_keys * (d_idx + 4.0) + len(lens) * G * d_idx * 1.0
    else:
        idx_bytes = scan_keys * d_idx * 2.0 + len(lens) * G * d_idx * 2.0
    idx_flops = 2.0 * d_idx * G * scan_keys
    keys = 0.0
    for b, L in enumerate(lens):
        for j in ids[b].ravel():
            if j >= 0:
                keys += min(block, int(L) - int(j) * block)
    attn_bytes = keys * d * 2.0 * 2.0  # K and V rows of each selected block, per group
    attn_flops = 4.0 * d * (H // G) * keys
    return dict(idx_bytes=idx_bytes, idx_flops=idx_flops, attn_bytes=attn_bytes,
                attn_flops=attn_flops, bytes=idx_bytes + attn_bytes)


# --------------------------------------------------------------------------
# environment helpers
# --------------------------------------------------------------------------

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            target = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", target, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, RuntimeError):
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        return self.parse_samples(out)

    @staticmethod
    def parse_samples(out: str) -> dict:
        """Median SM clock of the loaded samples (above half the highest seen), the
        maximum clock, and every throttle reason seen active in any sample."""
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        loaded = [c for c in sm if c > 0.5 * (max(sm) if sm else 0)]
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(init_group: bool = True):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and init_group:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local


def reduce_max(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def replica_rate(units_per_rank: float, ms_local: float, world: int):
    """Whole-job rate of `world` replicas that each processed `units_per_rank`
    units: the total over the slowest rank's time (max over ranks)."""
    ms = reduce_max(ms_local, world)
    return world * units_per_rank / (ms * 1e-3), ms


# --------------------------------------------------------------------------
# CPU oracle timing (the baseline arm)
# --------------------------------------------------------------------------

class OracleRows:
    """The oracle on sampled query rows of a prefill workload: the rows of q and
    q_idx are gathered where the inputs live and copied to the host, the key
    side (k, v, k_idx) is copied once."""

    def __init__(self, inp, shape):
        self.inp, self.shape = inp, shape
        self.key_side = {k: inp[k].cpu() for k in ("k", "v", "k_idx")}
        self.nb = (shape.N + shape.block - 1) // shape.block

    def gather(self, rows):
        ridx = torch.as_tensor(rows, device=self.inp["q"].device)
        return (self.inp["q"].index_select(0, ridx).cpu(),
                self.inp["q_idx"].index_select(0, ridx).cpu())

    def run(self, rows, q_rows, qi_rows):
        import oracle
        sh, ks = self.shape, self.key_side
        pooled = oracle.pooled_scores(qi_rows, rows, ks["k_idx"], sh.block, self.nb)
        ids = oracle.select_blocks(pooled, rows, sh.block, sh.top_k)
        return oracle.block_attention(q_rows, rows, ks["k"], ks["v"], ids, sh.scale, sh.block)


def oracle_prefill_rate(inp, shape, budget_s: float, max_rows: int = 4096, seed: int = 0):
    """Tokens/s of the oracle over a uniform sample of query rows."""
    orc = OracleRows(inp, shape)
    rows_done, elapsed, n = 0, 0.0, 16
    rng_seed = seed
    while elapsed < budget_s and rows_done < max_rows:
        rows = synth.sample_rows(shape.N, n, seed=rng_seed)[:n]
        rng_seed += 1
        q_rows, qi_rows = orc.gather(rows)
        t0 = time.perf_counter()
        orc.run(rows, q_rows, qi_rows)
        elapsed += time.perf_counter() - t0
        rows_done += len(rows)
        n = min(4 * n, max_rows - rows_done) if elapsed < budget_s / 4 else n
        if n <= 0:
            break
    return rows_done / elapsed, rows_done, elapsed


def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# --------------------------------------------------------------------------
# arms
# --------------------------------------------------------------------------

def run_reference(args, rank, world):
    if rank != 0:
        return None
    os.environ.setdefault("OMP_NUM_THREADS", str(cpu_cores()))
    shape = synth.PREFILL_CONFIGS[args.workload]
    # the seeded inputs are drawn where they are cheapest to draw (the device, if
    # any); only the sampled rows and the key side reach the oracle on the host
    inp = synth.make_prefill_inputs(shape, device="cuda" if torch.cuda.is_available() else "cpu")
    orc = OracleRows(inp, shape)
    rows_per_step = args.ref_rows
    step_times = []
    for i in range(args.warmup + args.steps):
        rows = synth.sample_rows(shape.N, rows_per_step, seed=1000 + i)[:rows_per_step]
        q_rows, qi_rows = orc.gather(rows)
        t0 = time.perf_counter()
        orc.run(rows, q_rows, qi_rows)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            step_times.append((dt, len(rows)))
    total_t = sum(t for t, _ in step_times)
    total_rows = sum(r for _, r in step_times)
    value = total_rows / total_t
    sample = (f"{rows_per_step} query rows per step, uniform over positions of the "
              f"{shape.name} workload (all heads and groups of each row)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total_t / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(args, shape),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": int(os.environ.get(
            "OMP_NUM_THREADS", cpu_cores())), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    return line


def decode_shape(args):
    return synth.DECODE_CONFIG if args.decode_workload == "full" else synth.DECODE_SMALL


def workload_config(args, shape):
    parts = [] if args.no_prefill else [shape.name]
    if not args.no_decode:
        parts.append(decode_shape(args).name)
    cfg = {"workload": "+".join(parts),
           "N": shape.N, "H": shape.H, "G": shape.G, "d": shape.d, "d_idx": shape.d_idx,
           "block": shape.block, "top_k": shape.top_k, "needles": shape.n_needles,
           "l2": "inputs larger than L2 (no flush)", "parallelism": "replicas",
           "index": "e4m3" if getattr(args, "index_fp8", False) else "bf16"}
    if getattr(args, "q8kv4", False):
        cfg["main_inputs"] = "MX: e4m3 q, e2m1 k/v, one E8M0 scale per 32 values"
    if not args.no_decode:
        dc = decode_shape(args)
        lens = sorted(set(dc.seq_lens))
        desc = "+".join(f"{dc.seq_lens.count(L)}x{L}" for L in lens)
        cfg["decode"] = {"seq_lens": desc, "B": dc.B, "H": dc.H, "G": dc.G, "d": dc.d,
                         "d_idx": dc.d_idx, "top_k": dc.top_k}
    return cfg


def _phase_ms(evs, n_phases):
    return [evs[i].elapsed_time(evs[i + 1]) for i in range(n_phases)]


class KernelTable:
    """Per-phase figures: mean event-timed ms, algorithmic work per launch, the
    achieved rate, and its fraction of the measured and of the nominal peak."""

    def __init__(self, peaks, tc_name, step_ms):
        self.peaks, self.tc_name, self.step_ms = peaks, tc_name, step_ms
        self.rows = {}

    def add(self, name, ms_arr, bound, work, peak_scale=1.0):
        ms = float(np.mean(ms_arr))
        if bound == "hbm":
            ach = work / (ms * 1e-3) / 1e9
            peak, nominal, unit = self.peaks["hbm_gbs"], NOMINAL_PEAKS["hbm_gbs"], "GB/s"
        else:
            ach = work / (ms * 1e-3) / 1e12
            peak = self.peaks[self.tc_name] * peak_scale
            nominal, unit = NOMINAL_PEAKS["bf16_tflops"] * peak_scale, "TFLOP/s"
        self.rows[name] = {"ms": ms, "ms_median": float(np.median(ms_arr)),
                           "ms_min": float(np.min(ms_arr)), "bound": bound, "achieved": ach,
                           "peak": peak, "unit": unit, "frac": ach / peak,
                           "frac_nominal": ach / nominal, "work_per_launch": work,
                           "share": ms / self.step_ms}
        return self.rows[name]


class PrefillRun:
    """One prefill workload on the device: inputs, workspace (capped; above the
    cap the query axis is processed in chunks) and the timed call."""

    def __init__(self, msa, shape, dev, rank, args):
        self.msa, self.shape, self.args = msa, shape, args
        N = shape.N
        self.cfg = msa.config(shape.H, shape.G, shape.d, shape.d_idx, top_k=shape.top_k,
                              block=shape.block, scale=shape.scale)
        self.inp = synth.make_prefill_inputs(shape, device=dev, seed=shape.seed + rank)
        q8kv4 = getattr(args, "q8kv4", False)
        full_ws = msa.msa_workspace_size(self.cfg, msa.OP_PREFILL, N)
        dq = (msa.msa_workspace_size(self.cfg, msa.OP_PREFILL_Q8KV4, N) - full_ws) if q8kv4 else 0
        cap = int(args.ws_gb * (1 << 30))
        self.ws = torch.empty(max(min(full_ws, cap), msa.msa_prefill_min_workspace(self.cfg, N))
                              + dq, dtype=torch.uint8, device=dev)
        self.out = torch.empty((N, shape.H, shape.d), dtype=torch.bfloat16, device=dev)
        self.ids = torch.empty((N, shape.G, shape.top_k), dtype=torch.int32, device=dev)
        chunk = msa.msa_prefill_chunk_tokens(self.cfg, N, self.ws.numel() - dq, ids_returned=True)
        self.n_chunks = (N + chunk - 1) // chunk
        self.quant_ms = None
        if args.index_fp8:
            # the quantised Index Branch takes e4m3 index tensors (a model with an
            # 8-bit indexer emits them from its projections): quantised once here,
            # the time reported beside the index kernel
            qz = msa.msa_quantize_index_fp8(self.cfg, self.inp["q_idx"], self.inp["k_idx"])
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            self.q8, self.k8, self.ks = msa.msa_quantize_index_fp8(self.cfg, self.inp["q_idx"],
                                                                   self.inp["k_idx"])
            e1.record()
            torch.cuda.synchronize()
            self.quant_ms = e0.elapsed_time(e1)
            del qz
        self.dq_start = []  # q8kv4: an event before each call (the dequantisation)
        if q8kv4:
            # MX inputs (a model serving a Q8KV4 cache holds them): quantised once
            # here, the quantiser's time reported beside the dequantisation
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            self.mx = (*msa.msa_quantize_mx(self.inp["q"], msa.MX_E4M3),
                       *msa.msa_quantize_mx(self.inp["k"], msa.MX_E2M1),
                       *msa.msa_quantize_mx(self.inp["v"], msa.MX_E2M1))
            e1.record()
            torch.cuda.synchronize()
            self.quant_ms = e0.elapsed_time(e1)

    def once(self):
        msa, inp = self.msa, self.inp
        if getattr(self.args, "q8kv4", False):
            ev = torch.cuda.Event(enable_timing=True)
            ev.record()
            self.dq_start.append(ev)
            q8, qs, k4, ks, v4, vs = self.mx
            msa.msa_prefill_q8kv4(self.cfg, q8, qs, k4, ks, v4, vs, inp["q_idx"], inp["k_idx"],
                                  out=self.out, ids_out=self.ids, workspace=self.ws)
        elif self.args.index_fp8:
            msa.msa_prefill_fp8_index(self.cfg, inp["q"], inp["k"], inp["v"], self.q8, self.k8,
                                      self.ks, out=self.out, ids_out=self.ids, workspace=self.ws)
        else:
            msa.msa_prefill(self.cfg, inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"],
                            out=self.out, ids_out=self.ids, workspace=self.ws)
        return msa.msa_last_launch_count()

    def events(self, steps):
        # 5 events per chunk of the query axis (phase boundaries)
        return [[torch.cuda.Event(enable_timing=True) for _ in range(5 * self.n_chunks)]
                for _ in range(steps)]

    def report(self, pev, table: KernelTable, world):
        """Phase times summed over the chunks of each step -> the prefill object;
        per-phase rows go into `table`."""
        shape, args = self.shape, self.args
        assert self.msa.msa_get_device_error(self.ws) == 0, "device error in timed prefill"
        nc = self.n_chunks
        pre_ph = np.array([[sum(e[5 * c + ph].elapsed_time(e[5 * c + ph + 1]) for c in range(nc))
                            for ph in range(4)] for e in pev])
        q8kv4 = getattr(args, "q8kv4", False)
        if q8kv4:  # the dequantisation runs before the library's first phase event
            starts = self.dq_start[-len(pev):]
            dq_ph = np.array([st.elapsed_time(e[0]) for st, e in zip(starts, pev)])
            pre_ph = np.concatenate([dq_ph[:, None], pre_ph], axis=1)
        value, pre_ms = replica_rate(shape.N, float(pre_ph.sum(axis=1).mean()), world)
        if q8kv4:
            N, H, G, d = shape.N, shape.H, shape.G, shape.d
            mx_bytes = (N * H * d * (1 + 2) + N * 2 * G * d * (0.5 + 2)
                        + (N * H + 2 * N * G) * d / 32)  # codes + scales in, bf16 out
            r = table.add("mx_dequantize", pre_ph[:, 0], "hbm", mx_bytes)
            r["quantize_ms"] = self.quant_ms
            pre_ph = pre_ph[:, 1:]
        pw = prefill_work(self.ids.cpu().numpy(), shape.H, shape.d, shape.block)
        idx_f = index_flops(shape.N, shape.G, shape.d_idx, shape.block)
        # e4m3 selection: its own dtype's peak, the measured bf16 one times the
        # nominal e4m3 / bf16 ratio (2)
        r = table.add("index_select", pre_ph[:, 0], "tensor", idx_f,
                      2.0 if args.index_fp8 else 1.0)
        if args.index_fp8:
            r["dtype"] = "e4m3"
            r["quantize_ms"] = self.quant_ms
        table.add("block_query_lists", pre_ph[:, 1], "hbm", pw["csr_bytes"])
        # the Main Branch against the tensor peak (its target); the HBM rate of its
        # algorithmic bytes beside it
        mb = table.add("main_branch", pre_ph[:, 2], "tensor", pw["main_flops"])
        mb["hbm_bytes_per_launch"] = pw["main_bytes"]
        mb["hbm_achieved_gbs"] = pw["main_bytes"] / (mb["ms"] * 1e-3) / 1e9
        mb["hbm_frac"] = mb["hbm_achieved_gbs"] / table.peaks["hbm_gbs"]
        table.add("merge", pre_ph[:, 3], "hbm", pw["merge_bytes"])
        return {"value": value, "unit": "tokens/s", "ms_per_step": pre_ms, "query_chunks": nc,
                "index_ms": float(pre_ph[:, 0].mean()),
                "main_ms": float(pre_ph[:, 1:].sum(axis=1).mean()),
                "index_flops": idx_f, "main_flops": pw["main_flops"],
                "dense_flops": dense_flops(shape.N, shape.H, shape.d),
                "msa_flops": idx_f + pw["main_flops"],
                "selected_keys_per_query": pw["selected_keys"]}


def _tc_peak_name(total_ms, step_ms):
    # the sustained (power-capped) bf16 figure for long steps or regions, the burst one else
    return "bf16_tflops_sustained" if (total_ms > 5000.0 or step_ms > 200.0) else "bf16_tflops"


def measure_extra(msa, name, args, dev, rank, world):
    """A prefill-only measurement of another workload (its own buffers, freed
    before return): prefill tokens/s, per-phase kernels and clocks."""
    shape = synth.PREFILL_CONFIGS[name]
    run = PrefillRun(msa, shape, dev, rank, args)
    steps = 20 if shape.N <= 65536 else 8
    for _ in range(3):
        run.once()
    torch.cuda.synchronize()
    assert msa.msa_get_device_error(run.ws) == 0, f"device error in {name} warm-up"
    pev = run.events(steps)
    barrier(world)
    torch.cuda.synchronize()
    sampler = ClockSampler(dev.index)
    time.sleep(0.3)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(steps):
        msa.msa_set_phase_events(pev[i])
        run.once()
    msa.msa_set_phase_events(None)
    t1.record()
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    total = reduce_max(t0.elapsed_time(t1), world)
    peaks, _ = load_peaks()
    table = KernelTable(peaks, _tc_peak_name(total, total / steps), total / steps)
    obj = run.report(pev, table, world)
    obj.update({"workload": name, "N": shape.N, "steps": steps, "warmup": 3,
                "kernels": table.rows, "clocks": clocks, "tc_peak": table.tc_name})
    del run
    torch.cuda.empty_cache()
    return obj


def measure_decode_alone(msa, dec, dcfg, dc, cu_dev, max_len, dws, dout, dids, args, world,
                         peaks, fp8: bool):
    """Decode tokens/s of decode steps run back to back (a decode serving loop),
    with the bf16 or the e4m3 Index Branch (per-row quantised index query and
    index-key cache; the attention reads the same bf16 K/V either way)."""
    if fp8:
        q8, _ = msa.msa_quantize_rows_fp8(dec["q_idx"])
        k8, ks = msa.msa_quantize_rows_fp8(dec["k_idx_cache"])

    def once():
        if fp8:
            msa.msa_decode_fp8_index(dcfg, dec["q"], q8, dec["k_cache"], dec["v_cache"], k8, ks,
                                     cu_dev, max_len, out=dout, ids_out=dids, workspace=dws)
        else:
            msa.msa_decode(dcfg, dec["q"], dec["q_idx"], dec["k_cache"], dec["v_cache"],
                           dec["k_idx_cache"], cu_dev, max_len, out=dout, ids_out=dids,
                           workspace=dws)

    for _ in range(3):
        once()
    torch.cuda.synchronize()
    assert msa.msa_get_device_error(dws) == 0, "device error in decode warm-up"
    steps = max(args.steps, 10)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    for i in range(steps):
        msa.msa_set_phase_events(evs[i])
        once()
    msa.msa_set_phase_events(None)
    torch.cuda.synchronize()
    barrier(world)
    ph = np.array([_phase_ms(e, 2) for e in evs])
    rate, ms = replica_rate(dc.B, float(ph.sum(axis=1).mean()), world)
    dw = decode_work(dc.seq_lens, dc.H, dc.G, dc.d, dc.d_idx, dids.cpu().numpy(), dc.block,
                     fp8_index=fp8)
    table = KernelTable(peaks, "bf16_tflops", ms)
    table.add("decode_index_fp8" if fp8 else "decode_index", ph[:, 0], "hbm", dw["idx_bytes"])
    table.add("decode_select_attend", ph[:, 1], "hbm", dw["attn_bytes"])
    if fp8:
        del q8, k8, ks
    return {"value": rate, "unit": "tokens/s", "ms_per_step": ms, "steps": steps,
            "bytes_per_step": dw["bytes"],
            "hbm_frac": dw["bytes"] / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
            "hbm_frac_nominal": dw["bytes"] / (ms * 1e-3) / 1e9 / NOMINAL_PEAKS["hbm_gbs"],
            "kernels": table.rows,
            "index": "e4m3, one fp32 scale per index-key row" if fp8 else "bf16"}


def run_ours(args, rank, world, local):
    import block_sparse_long_branch_b200 as msa
    dev = torch.device("cuda", local)
    shape = synth.PREFILL_CONFIGS[args.workload]
    do_prefill = not args.no_prefill
    N = shape.N
    run = PrefillRun(msa, shape, dev, rank, args) if do_prefill else None
    cfg = run.cfg if run else None

    dc = decode_shape(args)
    dec = None
    if not args.no_decode:
        dec = synth.make_decode_inputs(dc, device=dev, seed=dc.seed + rank)
        dcfg = msa.config(dc.H, dc.G, dc.d, dc.d_idx, top_k=dc.top_k, block=dc.block,
                          scale=dc.scale)
        cu_dev = dec["cu_seqlens"].to(dev)
        dws = torch.empty(msa.msa_workspace_size(dcfg, msa.OP_DECODE, dc.total_len, dc.B),
                          dtype=torch.uint8, device=dev)
        dout = torch.empty((dc.B, dc.H, dc.d), dtype=torch.bfloat16, device=dev)
        dids = torch.empty((dc.B, dc.G, dc.top_k), dtype=torch.int32, device=dev)
        max_len = max(dc.seq_lens)

    def decode_once():
        msa.msa_decode(dcfg, dec["q"], dec["q_idx"], dec["k_cache"], dec["v_cache"],
                       dec["k_idx_cache"], cu_dev, max_len, out=dout, ids_out=dids,
                       workspace=dws)
        return msa.msa_last_launch_count()

    # ---- warm-up ----
    for _ in range(args.warmup):
        if run:
            run.once()
        if dec is not None:
            decode_once()
    torch.cuda.synchronize()
    if run:
        assert msa.msa_get_device_error(run.ws) == 0, "device error after prefill warm-up"
    if dec is not None:
        assert msa.msa_get_device_error(dws) == 0, "device error after decode warm-up"

    pev = run.events(args.steps) if run else []
    dev_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    launches = 0
    barrier(world)
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    time.sleep(0.3)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record()
    for i in range(args.steps):
        if run:
            msa.msa_set_phase_events(pev[i])
            launches += run.once()
        if dec is not None:
            msa.msa_set_phase_events(dev_ev[i])
            launches += decode_once()
        msa.msa_set_phase_events(None)
    t_end.record()
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    total_ms = reduce_max(t_start.elapsed_time(t_end), world)
    step_ms = total_ms / args.steps
    peaks, peak_src = load_peaks()
    table = KernelTable(peaks, _tc_peak_name(total_ms, step_ms), step_ms)
    kernels = table.rows

    prefill_obj, value = None, None
    if run:
        prefill_obj = run.report(pev, table, world)
        value = prefill_obj["value"]
    decode_obj = None
    if dec is not None:
        dec_ph = np.array([_phase_ms(e, 2) for e in dev_ev])
        dec_rate, dec_ms = replica_rate(dc.B, float(dec_ph.sum(axis=1).mean()), world)
        dw = decode_work(dc.seq_lens, dc.H, dc.G, dc.d, dc.d_idx, dids.cpu().numpy(), dc.block)
        table.add("decode_index", dec_ph[:, 0], "hbm", dw["idx_bytes"])
        table.add("decode_select_attend", dec_ph[:, 1], "hbm", dw["attn_bytes"])
        dstep_bytes = dw["bytes"]
        decode_obj = {"value": dec_rate, "unit": "tokens/s",
                      "ms_per_step": dec_ms,
                      "hbm_frac": dstep_bytes / (dec_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                      "hbm_frac_nominal": dstep_bytes / (dec_ms * 1e-3) / 1e9 /
                      NOMINAL_PEAKS["hbm_gbs"],
                      "bytes_per_step": dstep_bytes}
        if value is None:
            value = decode_obj["value"]
        # decode steps back to back, as a decode serving loop runs them: in the
        # step above each decode follows a prefill, whose power-capped clock it
        # inherits
        decode_obj["alone"] = measure_decode_alone(msa, dec, dcfg, dc, cu_dev, max_len, dws,
                                                   dout, dids, args, world, peaks, fp8=False)
        # the same with the e4m3 Index Branch over an e4m3 index-key cache
        # (quantised once, before timing, as a model's projections would emit it)
        decode_obj["fp8_index"] = measure_decode_alone(msa, dec, dcfg, dc, cu_dev, max_len, dws,
                                                       dout, dids, args, world, peaks, fp8=True)
    dominant = max(kernels, key=lambda k: kernels[k]["ms"])
    dk = kernels[dominant]
    roofline = {"kernel": dominant, "bound": dk["bound"], "achieved": dk["achieved"],
                "peak": dk["peak"], "unit": dk["unit"], "frac": dk["frac"],
                "frac_nominal": dk["frac_nominal"],
                "traffic": traffic_for(dominant, shape.name if run else None),
                "peak_source": f"{peak_src} "
                f"({'hbm_gbs' if dk['unit'] == 'GB/s' else table.tc_name})"}

    # ---- end to end through the public API with host buffers ----
    e2e = None if (args.no_e2e or args.index_fp8 or args.q8kv4) else run_e2e(
        args, msa, cfg, shape, run.inp if run else None, run.ws if run else None,
        run.out if run else None, dev, dec, dcfg if dec is not None else None,
        dws if dec is not None else None, world)

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": workload_config(args, shape),
        "prefill": prefill_obj, "decode": decode_obj, "roofline": roofline, "kernels": kernels,
        "e2e": e2e, "gpu_launches": launches, "clocks": clocks,
    }
    if world == 1 and rank == 0 and run and not args.no_cpu_baseline:
        os.environ.setdefault("OMP_NUM_THREADS", str(cpu_cores()))
        rate, rows, el = oracle_prefill_rate(run.inp, shape, args.cpu_budget)
        line["cpu_baseline"] = {"value": rate, "unit": "tokens/s",
                                "cores": int(os.environ["OMP_NUM_THREADS"]), "kind": "oracle",
                                "sample": f"{rows} query rows uniform over the {shape.name} "
                                          f"positions, {el:.1f} s of oracle time"}
    extras = [x for x in (args.extra or "").split(",") if x and x != "none" and x != shape.name]
    if extras and world == 1:
        # the other prefill workloads, measured after this one's buffers are freed
        del run
        if dec is not None:
            del dec, dws, dout, dids
        torch.cuda.empty_cache()
        line["extra"] = {x: measure_extra(msa, x, args, dev, rank, world) for x in extras}
    return line


def traffic_for(kernel: str, workload):
    """DRAM bytes of one phase from a committed ncu summary, if it was captured on
    this workload and the kernel source is unchanged since (null otherwise)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            table = json.load(f)
    except (OSError, ValueError):
        return None
    ent = table.get(kernel)
    if not ent or ent.get("workload") != workload:
        return None
    src = os.path.join(ROOT, "block_sparse_long_branch_b200", "csrc", ent.get("source", ""))
    try:
        import hashlib
        with open(src, "rb") as f:
            h = hashlib.sha256(f.read()).hexdigest()[:16]
    except OSError:
        return None
    return ent.get("bytes_per_phase") if h == ent.get("source_sha") else None


def run_e2e(args, msa, cfg, shape, inp, ws, out, dev, dec, dcfg, dws, world):
    """Host (pinned) inputs -> device -> msa_prefill -> host output, every step.

    Up to 256K tokens, three streams overlap consecutive steps: step i's
    kernels run while step i+1's inputs are copied in and step i-1's output is
    copied out; inputs and outputs are double-buffered on both sides.  Beyond
    that (the 1M workload: 22 GB in and 16 GB out per step) the steps run one
    after another on one stream into the bench's own device buffers: copy in,
    prefill, copy out.  Either way each step moves its full inputs
    host->device and its full output device->host inside the timed region.
    """
    res = {}
    if inp is not None:
        if shape.N > (1 << 18):
            res = _e2e_prefill_serial(args, msa, cfg, shape, inp, ws, out, world)
        else:
            res = _e2e_prefill(args, msa, cfg, shape, inp, ws, dev, world)
    if dec is not None:
        res["decode"] = _e2e_decode(args, msa, dec, dcfg, dws, dev, world)
        if inp is None:
            res.update({k: v for k, v in res["decode"].items()})
    return res


def _e2e_prefill_serial(args, msa, cfg, shape, inp, ws, out, world):
    keys = ("q", "k", "v", "q_idx", "k_idx")
    host = {k: torch.empty_like(inp[k], device="cpu").pin_memory() for k in keys}
    for k in keys:
        host[k].copy_(inp[k])
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = sum(host[k].numel() * host[k].element_size() for k in keys)
    d2h = out_h.numel() * out_h.element_size()
    steps = max(2, min(args.steps, 3))

    def step():
        for k in keys:
            inp[k].copy_(host[k], non_blocking=True)
        msa.msa_prefill(cfg, inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"], out=out,
                        workspace=ws)
        out_h.copy_(out, non_blocking=True)

    step()
    torch.cuda.synchronize()
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        step()
    b.record()
    torch.cuda.synchronize()
    ms = reduce_max(a.elapsed_time(b) / steps, world)
    del host, out_h
    return {"value": world * shape.N / (ms * 1e-3), "unit": "tokens/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": ms,
            "steps": steps, "pipelined": "no: copy in, prefill, copy out on one stream"}


def _e2e_prefill(args, msa, cfg, shape, inp, ws, dev, world):
    keys = ("q", "k", "v", "q_idx", "k_idx")
    host = [{k: torch.empty_like(inp[k], device="cpu").pin_memory() for k in keys}
            for _ in range(2)]
    for hb in host:
        for k in keys:
            hb[k].copy_(inp[k])
    dbuf = [{k: torch.empty_like(inp[k]) for k in keys} for _ in range(2)]
    outs = [torch.empty((shape.N, shape.H, shape.d), dtype=torch.bfloat16, device=dev)
            for _ in range(2)]
    out_h = [torch.empty(outs[0].shape, dtype=outs[0].dtype).pin_memory() for _ in range(2)]
    h2d = sum(host[0][k].numel() * host[0][k].element_size() for k in keys)
    d2h = out_h[0].numel() * out_h[0].element_size()
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    steps = max(4, args.steps)

    def run(n, start=None, end=None):
        used = [False, False]
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_in):
                if used[b]:
                    s_in.wait_event(ev_cmp[b])  # buffer b's inputs consumed by step i-2
                if i == 0 and start is not None:
                    start.record(s_in)
                for k in keys:
                    dbuf[b][k].copy_(host[b][k], non_blocking=True)
                ev_in[b].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(ev_in[b])
                if used[b]:
                    s_cmp.wait_event(ev_out[b])  # output buffer b copied out by step i-2
                msa.msa_prefill(cfg, dbuf[b]["q"], dbuf[b]["k"], dbuf[b]["v"], dbuf[b]["q_idx"],
                                dbuf[b]["k_idx"], out=outs[b], workspace=ws, stream=s_cmp)
                ev_cmp[b].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_cmp[b])
                out_h[b].copy_(outs[b], non_blocking=True)
                ev_out[b].record(s_out)
            used[b] = True
        if end is not None:
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_in[(n - 1) % 2])
                end.record(s_out)

    run(2)
    torch.cuda.synchronize()
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    run(steps, a, b)
    torch.cuda.synchronize()
    ms = reduce_max(a.elapsed_time(b) / steps, world)
    res = {"value": world * shape.N / (ms * 1e-3), "unit": "tokens/s",
           "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": ms,
           "pipelined": "3 streams: copy-in, kernels, copy-out; double-buffered"}
    return res


def _e2e_decode(args, msa, dec, dcfg, dws, dev, world):
    dc = dec["shape"]
    steps = max(4, args.steps)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # per step: the new token's q / q_idx and its k, v, k_idx cache rows in,
    # the attention output back
    last = (dec["cu_seqlens"][1:] - 1).to(dev)
    hq = dec["q"].cpu().pin_memory()
    hqi = dec["q_idx"].cpu().pin_memory()
    hk = dec["k_cache"][last].cpu().pin_memory()
    hv = dec["v_cache"][last].cpu().pin_memory()
    hki = dec["k_idx_cache"][last].cpu().pin_memory()
    dq, dqi = torch.empty_like(dec["q"]), torch.empty_like(dec["q_idx"])
    drow_k, drow_v, drow_ki = (torch.empty_like(hk, device=dev),
                               torch.empty_like(hv, device=dev),
                               torch.empty_like(hki, device=dev))
    dout = torch.empty((dc.B, dc.H, dc.d), dtype=torch.bfloat16, device=dev)
    dout_h = torch.empty(dout.shape, dtype=dout.dtype).pin_memory()
    cu_dev = dec["cu_seqlens"].to(dev)
    dh2d = sum(x.numel() * x.element_size() for x in (hq, hqi, hk, hv, hki))

    def dstep():
        dq.copy_(hq, non_blocking=True)
        dqi.copy_(hqi, non_blocking=True)
        drow_k.copy_(hk, non_blocking=True)
        drow_v.copy_(hv, non_blocking=True)
        drow_ki.copy_(hki, non_blocking=True)
        dec["k_cache"].index_copy_(0, last, drow_k)
        dec["v_cache"].index_copy_(0, last, drow_v)
        dec["k_idx_cache"].index_copy_(0, last, drow_ki)
        msa.msa_decode(dcfg, dq, dqi, dec["k_cache"], dec["v_cache"], dec["k_idx_cache"],
                       cu_dev, max(dc.seq_lens), out=dout, workspace=dws)
        dout_h.copy_(dout, non_blocking=True)

    for _ in range(2):
        dstep()
    torch.cuda.synchronize()
    a.record()
    for _ in range(steps):
        dstep()
    b.record()
    torch.cuda.synchronize()
    dms = reduce_max(a.elapsed_time(b) / steps, world)
    return {"value": world * dc.B / (dms * 1e-3), "unit": "tokens/s",
            "h2d_bytes_per_step": int(dh2d),
            "d2h_bytes_per_step": int(dout_h.numel() * dout_h.element_size()),
            "ms_per_step": dms}


def run_varlen(args, rank, world, local):
    """A packed batch of equal-length sequences: the one-pass varlen prefill
    against one msa_prefill per sequence, both timed with CUDA events."""
    import block_sparse_long_branch_b200 as msa
    B, L = (int(x) for x in args.varlen.lower().split("x"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    msa.load_library()
    cu = np.arange(B + 1, dtype=np.int64) * L
    shape = synth.PrefillShape(f"varlen_{B}x{L}", N=B * L, H=64, G=8, d=128, d_idx=128,
                               top_k=16, seed=synth.SEED_BASE + 40)
    inp = synth.make_prefill_inputs(shape, device=dev, seed=shape.seed + rank)
    cfg = msa.config(shape.H, shape.G, shape.d, shape.d_idx, top_k=shape.top_k,
                     scale=shape.scale)
    ws = torch.empty(msa.msa_prefill_varlen_workspace_size(cfg, cu), dtype=torch.uint8,
                     device=dev)
    out = torch.empty((shape.N, shape.H, shape.d), dtype=torch.bfloat16, device=dev)
    ref = torch.empty_like(out)

    def one_pass():
        msa.msa_prefill_varlen(cfg, inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"], cu,
                               out=out, workspace=ws)

    def per_sequence():
        for b in range(B):
            r = slice(b * L, (b + 1) * L)
            msa.msa_prefill(cfg, inp["q"][r], inp["k"][r], inp["v"][r], inp["q_idx"][r],
                            inp["k_idx"][r], out=ref[r], workspace=ws)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        barrier(world)
        return reduce_max(e0.elapsed_time(e1), world) / args.steps

    ms_one = timed(one_pass)
    ms_seq = timed(per_sequence)
    assert torch.equal(out, ref), "one pass and per-sequence prefill differ"
    value, _ = replica_rate(shape.N, ms_one, world)
    return {"metric": "MSA varlen prefill tokens/s (one pass over the packed batch)",
            "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_one, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": shape.name, "B": B, "L": L, "H": shape.H, "G": shape.G,
                       "d": shape.d, "d_idx": shape.d_idx, "top_k": shape.top_k},
            "per_sequence_ms": ms_seq, "speedup_vs_per_sequence": ms_seq / ms_one}


def run_phase(args, rank, world, local):
    """Only one phase of the prefill, on the workload's tensors: the Index Branch
    selection (msa_select_topk) or the query-list build (msa_build_block_query_lists
    on that selection).  For profiling one kernel on a small device footprint."""
    import block_sparse_long_branch_b200 as msa
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    shape = synth.PREFILL_CONFIGS[args.workload]
    inp = synth.make_prefill_inputs(shape, device=dev, seed=shape.seed + rank)
    for k in ("q", "k", "v"):
        del inp[k]
    torch.cuda.empty_cache()
    cfg = msa.config(shape.H, shape.G, shape.d, shape.d_idx, top_k=shape.top_k,
                     block=shape.block, scale=shape.scale)
    N = shape.N
    ids = torch.empty((N, shape.G, shape.top_k), dtype=torch.int32, device=dev)
    sws = torch.empty(msa.msa_workspace_size(cfg, msa.OP_SELECT_TOPK, N), dtype=torch.uint8,
                      device=dev)
    lws = torch.empty(msa.msa_workspace_size(cfg, msa.OP_BLOCK_QUERY_LISTS, N), dtype=torch.uint8,
                      device=dev)
    msa.msa_select_topk(cfg, inp["q_idx"], inp["k_idx"], ids=ids, workspace=sws)

    def once():
        if args.phase == "select":
            msa.msa_select_topk(cfg, inp["q_idx"], inp["k_idx"], ids=ids, workspace=sws)
        else:
            msa.msa_build_block_query_lists(cfg, ids, workspace=lws)

    for _ in range(args.warmup):
        once()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        once()
    e1.record()
    torch.cuda.synchronize()
    ms = reduce_max(e0.elapsed_time(e1), world) / args.steps
    peaks, _ = load_peaks()
    if args.phase == "select":
        work, unit, peak = index_flops(N, shape.G, shape.d_idx, shape.block) / (ms * 1e-3) / 1e12, \
            "TFLOP/s", peaks["bf16_tflops"]
    else:
        work, unit, peak = 3.0 * N * shape.G * shape.top_k * 4.0 / (ms * 1e-3) / 1e9, "GB/s", \
            peaks["hbm_gbs"]
    return {"metric": f"MSA {args.phase} phase alone", "value": world * N / (ms * 1e-3),
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic", "config": {"workload": shape.name},
            "achieved": work, "achieved_unit": unit, "frac": work / peak}


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: 10 for the 1M workload, 20 otherwise)")
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.PREFILL_CONFIGS))
    ap.add_argument("--extra", default=DEFAULT_EXTRA,
                    help="comma-separated prefill workloads measured after the main one "
                         "(prefill only, own buffers, one GPU); 'none' to skip")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-prefill", action="store_true",
                    help="time only the decode step (profiling)")
    ap.add_argument("--decode-workload", choices=("full", "small"), default="full")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--index-fp8", action="store_true",
                    help="prefill with the quantised (e4m3) Index Branch; e2e is not run")
    ap.add_argument("--q8kv4", action="store_true",
                    help="prefill on MX inputs (e4m3 q, e2m1 k/v): msa_prefill_q8kv4; e2e is "
                         "not run")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the host-buffer end-to-end leg (large workloads)")
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of oracle time for the cpu_baseline sample")
    ap.add_argument("--ws-gb", type=float, default=96.0,
                    help="cap on the prefill workspace; above it the query axis is chunked")
    ap.add_argument("--ref-rows", type=int, default=32,
                    help="query rows per step in the reference arm")
    ap.add_argument("--phase", choices=("select", "lists"),
                    help="time only the Index Branch selection or only the query-list build "
                         "on the workload's index tensors (profiling)")
    ap.add_argument("--varlen", metavar="BxL",
                    help="time only a packed batch of B sequences of L tokens (64 heads, 8 "
                         "groups, d 128): one msa_prefill_varlen pass vs one msa_prefill "
                         "per sequence")
    args = ap.parse_args(argv)
    if args.steps is None:
        args.steps = 10 if synth.PREFILL_CONFIGS[args.workload].N > (1 << 18) else 20
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be >= 3")
    return args


def main(argv=None):
    args = parse_args(argv)
    rank, world, local = dist_setup(init_group=args.impl == "ours")
    if args.gpus != world and world > 1:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    try:
        if args.impl == "reference":
            line = run_reference(args, rank, world)
        elif args.varlen:
            line = run_varlen(args, rank, world, local)
        elif args.phase:
            line = run_phase(args, rank, world, local)
        else:
            line = run_ours(args, rank, world, local)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            if dist.is_available() and dist.is_initialized():
                dist.destroy_process_group()


if __name__ == "__main__":
    main()
