"""Paged attention benchmark on B200: KV-read GB/s, decode seqs/s, roofline fraction.

Decode (default).  One step = one decode step of the whole hot path for one batch:
  cache append (pa_reshape_and_cache) -> [copy-on-write copies] -> pa_decode
  (split-K partition kernel + merge kernel), or pa_decode_shared_prefix for the
  shared-prefix workload
on a synthetic workload (default: Llama-3-8B-shaped GQA decode, 128 sequences,
32 q / 8 kv heads, head_dim 128, block 16, bf16, context lens uniform in
[1024, 8192], shuffled physical blocks; --config / --workload pick another).
The KV cache (2.5 GB) is larger than L2, so no flush is needed between steps.

Prefill (--op prefill).  One step = append the chunks' K, V, then pa_prefill;
metric TFLOP/s of causal attention against the measured bf16 tensor peak.

Printed (rank 0, one JSON line):
  value   -- algorithmic bytes (or FLOPs) per step / device step time (CUDA events)
  e2e     -- the same metric through the public API with host buffers: host
             pool appends + table packing, H2D of the step's inputs, the step,
             D2H of the output, every step (pipelined over two staging slots)
  roofline -- the attention call's algorithmic bytes (FLOPs) / its measured
             launch time against the measured HBM copy bandwidth (bf16 peak),
             with the DRAM traffic of the committed ncu capture
  cpu_baseline -- the fp64 oracle on the host cores over a bounded sample
  clocks  -- SM clock and throttle reasons sampled inside the timed region

--impl reference runs the oracle (the only reference this method has here) on
a bounded sample of the same workload on the host cores.
With torchrun (decode), the N ranks split one global batch of N x the
workload's sequences by sequence (pa_plan_shards: longest first, to the rank
with the fewest tokens; decode needs no data exchange between ranks), each
rank running its share on its own GPU; prefill runs N independent replicas.
value = the units all ranks processed / max time over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time


def _nvml_sampler(pci_id: str, path: str) -> None:
    """Child process: append "wall_time sm_mhz max_mhz reason_bits" every ~1 ms."""
    import pynvml as nv
    nv.nvmlInit()
    h = nv.nvmlDeviceGetHandleByPciBusId(pci_id) if pci_id else nv.nvmlDeviceGetHandleByIndex(0)
    mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
    with open(path, "w", buffering=1) as f:
        while True:
            try:
                f.write(f"{time.time():.6f} {nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)} {mx} "
                        f"{int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))}\n")
            except Exception:
                pass
            time.sleep(0.001)


if __name__ == "__main__" and len(sys.argv) == 4 and sys.argv[1] == "--nvml-sampler":
    _nvml_sampler(sys.argv[2], sys.argv[3])        # clock-sampling child (no torch import)
    sys.exit(0)

import torch  # noqa: E402

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)
# raw clock logs (the JSON line carries their summary); PA_BENCH_LOG_DIR overrides
LOG_DIR = os.environ.get("PA_BENCH_LOG_DIR", os.path.join(ROOT, "bench_logs"))

import workloads as wl  # noqa: E402

METRIC = "paged decode KV-read GB/s (% of B200 HBM peak) and decode seqs/s"
# the other multi-sequence decode workloads the default run also times (device only)
EXTRA_WORKLOADS = ("llama2_7b_mha_fp16_b64", "long_context_splitk_bf16_4x100k",
                   "prefix_shared_fp8_b256")
FALLBACK_HBM_GBS = 6650.0


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def _reduce(x: float, dev, op) -> float:
    """x combined over the ranks of the default process group (x itself when
    there is none); dev is where the backend takes tensors (cuda for NCCL,
    cpu for gloo)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(x: float, dev) -> float:
    return _reduce(x, dev, torch.distributed.ReduceOp.MAX)


def sum_over_ranks(x: float, dev) -> float:
    return _reduce(x, dev, torch.distributed.ReduceOp.SUM)


def whole_job_rate(units: float, ms: float, dev) -> float:
    """Units all ranks processed per second, over the slowest rank's time: each
    replica draws its own inputs, so the units differ from rank to rank."""
    return sum_over_ranks(units, dev) / (max_over_ranks(ms, dev) * 1e-3)


def algorithmic_bytes(cfg: wl.DecodeConfig, lens: torch.Tensor) -> dict:
    """Bytes the step must move at minimum (no tail slots, no split-K partials)."""
    e_kv, e_q = wl.elem_bytes(cfg.kv_dtype), wl.elem_bytes(cfg.q_dtype)
    S, Hq, Hkv, D, bs = cfg.num_seqs, cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim, cfg.block_size
    n = lens.to(torch.int64)
    kv = int(n.sum()) * Hkv * D * 2 * e_kv
    qo = S * Hq * D * 2 * e_q
    tables = int(((n + bs - 1) // bs).sum()) * 4 + S * 4
    decode = kv + qo + tables
    append = S * Hkv * D * 2 * (e_q + e_kv) + S * 8
    # with a shared prefix every sequence reads the same prefix blocks: count them once
    unique_kv = kv - max(S - 1, 0) * cfg.prefix_tokens * Hkv * D * 2 * e_kv
    return {"decode": decode, "append": append, "kv": kv, "unique_kv": unique_kv,
            "decode_unique": unique_kv + qo + tables}


def _pci_id(dev: int) -> str | None:
    p = torch.cuda.get_device_properties(dev)
    try:
        return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
    except AttributeError:
        return None


class ClockSampler:
    """SM clock and clock-event reasons sampled DURING the timed region.

    A child process polls NVML about every millisecond and timestamps each
    sample (a decode step is well under a millisecond, and a thread in this
    process would be starved by the launch loop); samples inside
    [mark_start, mark_end] are kept.  nvidia-smi's own log runs beside it as
    the raw record.  Read-only queries: nothing on the GPU is changed.
    """
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, dev: int):
        self.t0 = self.t1 = None
        pid = _pci_id(dev)
        os.makedirs(LOG_DIR, exist_ok=True)
        self.path = os.path.join(LOG_DIR, f"nvml_rank{dev}.log")
        if os.path.exists(self.path):      # a previous run's log would end the wait below early
            os.remove(self.path)
        self.child = subprocess.Popen([sys.executable, os.path.abspath(__file__),
                                       "--nvml-sampler", pid or "", self.path],
                                      stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        self.proc = None
        try:
            args = ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                    "-lms", "200"] + (["-i", pid] if pid else [])
            self.f = open(os.path.join(LOG_DIR, f"clocks_rank{dev}.csv"), "w")
            self.proc = subprocess.Popen(args, stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        # wait until the child has produced its first sample
        for _ in range(1500):
            if os.path.exists(self.path) and os.path.getsize(self.path) > 0:
                break
            time.sleep(0.01)

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self) -> dict:
        time.sleep(0.01)
        for p in (self.child, self.proc):
            if p is None:
                continue
            p.terminate()
            try:
                p.wait(timeout=5)
            except Exception:
                p.kill()
        if self.proc is not None:
            self.f.close()
        import pynvml as nv
        names = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                 "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                 "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                 "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap,
                 "hw_power_brake_slowdown": nv.nvmlClocksEventReasonHwPowerBrakeSlowdown}
        sm, mx, bits = [], None, 0
        try:
            for line in open(self.path):
                c = line.split()
                if len(c) != 4:
                    continue
                t = float(c[0])
                if self.t0 is not None and self.t0 <= t <= self.t1:
                    sm.append(float(c[1]))
                    mx = float(c[2])
                    bits |= int(c[3])
        except OSError:
            pass
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": ["unsampled"]}
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": mx,
                "reasons": sorted(n for n, b in names.items() if bits & b),
                "samples": len(sm), "sm_mhz_min": sm[0], "source": "nvml child process, 1 ms"}


# ------------------------------------------------------------------ oracle arm

def _sample_cfg(cfg: wl.DecodeConfig, nseq: int) -> wl.DecodeConfig:
    """nseq sequences drawn like the workload's (same heads, dtypes, lengths)."""
    import dataclasses
    nseq = max(1, min(nseq, cfg.num_seqs))
    if cfg.fixed_lens:
        return dataclasses.replace(cfg, num_seqs=nseq, fixed_lens=cfg.fixed_lens[:nseq],
                                   fixed_num_blocks=None, name=cfg.name + f"_sample{nseq}")
    if cfg.prefix_tokens:
        return wl.small_variant(cfg, nseq, cfg.suffix_lo, cfg.suffix_hi)
    return wl.small_variant(cfg, nseq, cfg.ctx_lo, cfg.ctx_hi)


def _oracle_pass(inp: wl.DecodeInputs, cores: int) -> float:
    import oracle  # test infrastructure: only the CPU-baseline / reference legs use it
    c = inp.cfg
    t0 = time.perf_counter()
    oracle.paged_decode(inp.q, c.q_dtype, inp.key_cache, inp.value_cache, c.kv_dtype,
                        inp.block_tables, inp.context_lens, inp.scale, inp.k_scale, inp.v_scale,
                        nthreads=cores)
    return time.perf_counter() - t0


def oracle_sample(cfg: wl.DecodeConfig, seed: int, pass_s: float):
    """A sample sized so one oracle pass takes about pass_s seconds."""
    cores = os.cpu_count() or 1
    probe = wl.make_decode_inputs(_sample_cfg(cfg, 1), seed=seed)
    t1 = max(_oracle_pass(probe, cores), 1e-3)
    # one sequence occupies at most Hkv threads; more sequences fill the rest
    per_seq = t1 / max(1.0, min(cores, cfg.num_kv_heads) / cfg.num_kv_heads * 1.0)
    nseq = int(max(1, min(cfg.num_seqs, pass_s / per_seq * max(1, cores // cfg.num_kv_heads))))
    return wl.make_decode_inputs(_sample_cfg(cfg, nseq), seed=seed), cores


def cpu_oracle_rate(cfg: wl.DecodeConfig, seed: int, budget_s: float = 15.0) -> dict:
    """The fp64 oracle on the host cores over a bounded sample of the workload."""
    inp, cores = oracle_sample(cfg, seed, budget_s / 2)
    t, reps = 0.0, 0
    while reps < 1 or t < budget_s / 2:
        t += _oracle_pass(inp, cores)
        reps += 1
    kv = algorithmic_bytes(inp.cfg, inp.context_lens)["kv"]
    S = inp.cfg.num_seqs
    return {"gbs": kv * reps / t / 1e9, "seqs_per_s": S * reps / t, "cores": cores,
            "seconds": t / reps,
            "sample": f"{S} sequences drawn like the workload's ({kv / 1e9:.3f} GB of K/V), "
                      f"fp64 oracle on {cores} threads, {reps} passes"}


def run_reference(args, cfg, rank, world):
    if rank != 0:
        return
    budget = max(1.0, 150.0 / (args.warmup + args.steps))   # whole run within a few minutes
    inp, cores = oracle_sample(cfg, args.seed, budget)
    for _ in range(args.warmup):
        _oracle_pass(inp, cores)
    ts = [_oracle_pass(inp, cores) for _ in range(args.steps)]
    kv = algorithmic_bytes(inp.cfg, inp.context_lens)["kv"]
    sec = sum(ts) / len(ts)
    gbs = kv / sec / 1e9
    sample = (f"{inp.cfg.num_seqs} sequences drawn like the workload's ({kv / 1e9:.3f} GB of K/V) "
              f"per step, fp64 oracle on {cores} threads")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * sec, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _config_dict(cfg, args),
        "seqs_per_s": round(inp.cfg.num_seqs / sec, 3),
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _config_dict(cfg, args, partition=None, l2_note=None):
    d = {"workload": cfg.name, "num_seqs": cfg.num_seqs, "q_heads": cfg.num_q_heads,
         "kv_heads": cfg.num_kv_heads, "head_dim": cfg.head_dim, "block_size": cfg.block_size,
         "kv_dtype": cfg.kv_dtype, "q_dtype": cfg.q_dtype,
         "context_lens": list(cfg.fixed_lens[:1]) * 1 if cfg.fixed_lens else [cfg.ctx_lo, cfg.ctx_hi],
         "parallelism": f"seq-shards{args.gpus}" if args.gpus > 1 else "single"}
    if cfg.prefix_tokens:
        d.update(prefix_tokens=cfg.prefix_tokens, suffix=[cfg.suffix_lo, cfg.suffix_hi])
    if partition is not None:
        d["partition"] = partition
    if l2_note:
        d["l2"] = l2_note
    return d


# --------------------------------------------------------------------- GPU arm

def _traffic(cfg, part, shared):
    """DRAM read + write bytes of one attention call from the committed ncu
    capture of the same workload and path (profiles/traffic_<workload>[_shared_prefix].json),
    or None when there is none, it was taken for another partition, or it does
    not carry the hash of the kernel sources it was taken on (a capture of
    kernels that have changed since says nothing about the ones timed)."""
    name = f"traffic_{cfg.name}{'_shared_prefix' if shared else ''}.json"
    pj = _committed_capture(name)
    if pj is None or (not shared and pj.get("partition") != part):
        return None
    return pj.get("dram_bytes_per_launch")


def _committed_capture(name):
    """The profiles/<name> traffic record if it was taken on the current kernel
    sources (its csrc_sha256 equals csrc_sha256()), else None."""
    prof = os.path.join(ROOT, "profiles", name)
    if not os.path.exists(prof):
        return None
    try:
        with open(prof) as f:
            pj = json.load(f)
    except Exception:
        return None
    if pj.get("csrc_sha256") != csrc_sha256():
        return None
    return pj


def csrc_sha256() -> str:
    """Hash of the library's CUDA sources and headers under csrc/ (the .cu,
    .cuh and .h files: kernels and their launches; the host-only .cpp files
    do not change what a kernel reads)."""
    import hashlib
    d = os.path.join(ROOT, "paged_kv_cache_338_b200", "csrc")
    h = hashlib.sha256()
    for fn in sorted(os.listdir(d)):
        if not fn.endswith((".cu", ".cuh", ".h")):
            continue
        with open(os.path.join(d, fn), "rb") as f:
            h.update(fn.encode() + b"\0" + f.read())
    return h.hexdigest()


def device_leg(args, cfg, pa, dev, seed, steps, warmup, partition=-1):
    """Append [+ copy-on-write] + decode on device-resident inputs: W untimed
    steps, then K steps timed with CUDA events on the launching stream, clocks
    sampled inside the timed region.  The timed steps replay the step's kernels
    from CUDA graphs (unless --no-graph); 20 eagerly launched steps are timed
    before them for comparison."""
    stream = torch.cuda.current_stream()
    inp = wl.make_decode_inputs(cfg, seed=seed, device=dev)
    S, Hq, D = inp.q.shape
    part = partition if partition >= 0 else (
        cfg.partition or pa.pa_decode_suggest_partition(cfg.num_kv_heads, cfg.block_size,
                                                        inp.context_lens.cpu()))
    max_ctx = inp.max_ctx
    shared = bool(cfg.prefix_tokens) and not args.no_shared_prefix
    if shared:      # the batch's tables start with the same prefix blocks
        ws_bytes = pa.pa_decode_shared_prefix_workspace_size(
            S, Hq, cfg.num_kv_heads, D, cfg.block_size, max_ctx, cfg.prefix_tokens,
            inp.key_cache.dtype)
        part = 0
    else:
        ws_bytes = pa.pa_decode_workspace_size(S, Hq, D, max_ctx, part)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    out = torch.empty_like(inp.q)
    kc, vc = inp.key_cache, inp.value_cache
    pairs = inp.copy_pairs
    nbytes = algorithmic_bytes(cfg, inp.context_lens.cpu())

    def decode(out_t, q_t, tables, lens):
        if shared:
            pa.pa_decode_shared_prefix(out_t, q_t, kc, vc, tables, lens, max_ctx, inp.scale,
                                       cfg.prefix_tokens, ws if ws_bytes else None,
                                       inp.k_scale, inp.v_scale)
        else:
            pa.pa_decode(out_t, q_t, kc, vc, tables, lens, max_ctx, inp.scale, inp.k_scale,
                         inp.v_scale, part, ws if ws_bytes else None)

    def append():
        if pairs.numel():
            pa.pa_copy_blocks(kc, vc, pairs)
        pa.pa_reshape_and_cache(inp.key_new, inp.value_new, kc, vc, inp.slot_mapping,
                                inp.k_scale, inp.v_scale)

    graphs = None

    def step(ev=None):
        if ev is not None:
            ev[2].record(stream)
        if graphs:
            graphs[0].replay()
        else:
            append()
        if ev is not None:
            ev[0].record(stream)
        if graphs:
            graphs[1].replay()
        else:
            decode(out, inp.q, inp.block_tables, inp.context_lens)
        if ev is not None:
            ev[1].record(stream)

    # copy-on-write, append, then the decode's kernels (counted by the library)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    assert pa.pa_device_status() == 0
    n0 = pa.pa_launch_count()
    step()
    torch.cuda.synchronize()
    launches_per_step = pa.pa_launch_count() - n0

    def timed(nsteps):
        evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(nsteps)]
        for i in range(nsteps):
            step(evs[i])
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b, _ in evs) / nsteps

    # The decode step as a serving loop runs it: the same kernels launched from
    # two CUDA graphs (append + copy-on-write, decode) captured once, so the
    # timed region measures the GPU's work rather than the host's launch rate.
    # The eagerly launched step is timed beside it (decode_ms_eager).
    eager_dec = timed(min(steps, 20))
    graph_note = None
    if not args.no_graph:
        try:
            cap = [torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()]
            with torch.cuda.graph(cap[0]):
                append()
            with torch.cuda.graph(cap[1]):
                decode(out, inp.q, inp.block_tables, inp.context_lens)
            graphs = cap
            for _ in range(warmup):
                step()
            torch.cuda.synchronize()
            assert pa.pa_device_status() == 0
        except RuntimeError as e:      # capture refused: time the eager loop
            graphs = None
            graph_note = f"eager (graph capture failed: {str(e).splitlines()[0][:120]})"
            torch.cuda.synchronize()

    dist = torch.distributed.is_available() and torch.distributed.is_initialized()
    if dist:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(dev.index or 0)
    evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks.mark_start()
    t0.record(stream)
    for i in range(steps):
        step(evs[i])
    t1.record(stream)
    torch.cuda.synchronize()
    clocks.mark_end()
    clk = clocks.stop()
    assert pa.pa_device_status() == 0
    if dist:
        torch.distributed.barrier()
    dec_ms = [a.elapsed_time(b) for a, b, _ in evs]
    res = {"ms": t0.elapsed_time(t1), "dec_avg": sum(dec_ms) / len(dec_ms),
           "dec_eager": eager_dec,
           "launch": "cuda graph" if graphs else (graph_note or "eager"),
           "app_avg": sum(c.elapsed_time(a) for a, _, c in evs) / len(evs),
           "nbytes": nbytes, "part": part, "shared": shared, "S": S,
           "launches_per_step": launches_per_step, "clocks": clk,
           "kv_gb": nbytes["kv"] / 1e9}
    del graphs, inp, ws, out, kc, vc
    torch.cuda.empty_cache()
    return res


def roofline_of(cfg, r, peak, peak_kind):
    """The attention call against the HBM roofline.  With a shared prefix the
    algorithmic bytes count the prefix once (it is the same physical blocks for
    every sequence); logical bytes, which count it per sequence, are reported
    beside it and are no HBM fraction."""
    nb, t = r["nbytes"], r["dec_avg"] * 1e-3
    alg = nb["decode_unique"] if r["shared"] else nb["decode"]
    achieved = alg / t / 1e9
    d = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
         "frac": round(achieved / peak, 4), "traffic": _traffic(cfg, r["part"], r["shared"]),
         "peak_kind": peak_kind, "algorithmic_bytes": alg,
         "kernel": "pa_decode_shared_prefix (prefix records + suffix decode)"
         if r["shared"] else "pa_decode (partition + merge)"}
    if r["shared"]:
        d["logical_gbs_not_hbm"] = round(nb["decode"] / t / 1e9, 1)
    return d


def sharded_cfg(cfg, seed, rank, world, pa):
    """This rank's share of one global batch: world x num_seqs sequences drawn
    like the workload's (the same draw on every rank), split by sequence with
    pa_plan_shards (longest first, to the least loaded rank), so every rank
    streams about the same K/V and no rank waits on another's data."""
    if world == 1:
        return cfg
    import dataclasses
    g = dataclasses.replace(cfg, num_seqs=cfg.num_seqs * world, fixed_num_blocks=None,
                            fixed_lens=tuple(cfg.fixed_lens) * world if cfg.fixed_lens else None)
    lens = wl.draw_context_lens(g, seed)
    dev_of, _ = pa.pa_plan_shards(lens, world)
    mine = lens[dev_of.to(torch.int64) == rank]
    return dataclasses.replace(cfg, num_seqs=int(mine.numel()), fixed_lens=tuple(mine.tolist()),
                               fixed_num_blocks=None, name=f"{cfg.name}_shard{rank}of{world}")


def run_gpu(args, cfg, rank, world, local_rank):
    import paged_kv_cache_338_b200 as pa
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    if args.decode_select is not None:
        pa.pa_decode_select(args.decode_select)
    shard = sharded_cfg(cfg, args.seed, rank, world, pa)     # the workload itself at N = 1
    r = device_leg(args, shard, pa, dev, args.seed + rank, args.steps, args.warmup, args.partition)
    S, part, nbytes = r["S"], r["part"], r["nbytes"]
    step_bytes = nbytes["decode"] + nbytes["append"]
    value = whole_job_rate(step_bytes * args.steps, r["ms"], dev) / 1e9
    ms = max_over_ranks(r["ms"], dev)
    ms_step = ms / args.steps
    seqs_all = sum_over_ranks(S, dev)

    # ---- end to end through the public API with host buffers -------------
    e2e = run_e2e(args, shard, pa, dev, part) if not args.no_e2e else None
    if e2e is not None:
        e2e["value"] = whole_job_rate(e2e["bytes"], e2e["ms"], dev) / 1e9

    # ---- the other multi-sequence decode workloads, device-timed only ------
    extras = {}
    if args.workloads_also:
        for name in args.workloads_also.split(","):
            wcfg = wl.DECODE_WORKLOADS[name]
            x = device_leg(args, sharded_cfg(wcfg, args.seed, rank, world, pa), pa, dev,
                           args.seed + rank, args.steps, args.warmup)
            xv = whole_job_rate((x["nbytes"]["decode"] + x["nbytes"]["append"]) * args.steps,
                                x["ms"], dev) / 1e9
            extras[name] = (wcfg, x, xv, max_over_ranks(x["ms"], dev) / args.steps)

    if rank != 0:
        return
    peak, peak_kind = _peaks()
    roof = roofline_of(cfg, r, peak, peak_kind)
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        c = cpu_oracle_rate(cfg, args.seed, budget_s=args.cpu_budget)
        cpu = {"value": round(c["gbs"], 4), "unit": "GB/s", "cores": c["cores"],
               "kind": "oracle", "sample": c["sample"], "seqs_per_s": round(c["seqs_per_s"], 3)}
    workloads = {}
    for name, (wcfg, x, xv, xms) in extras.items():
        workloads[name] = {
            "value": round(xv, 2), "unit": "GB/s", "ms_per_step": round(xms, 4),
            "decode_ms": round(x["dec_avg"], 4), "decode_ms_eager": round(x["dec_eager"], 4),
            "launch": x["launch"], "append_cow_ms": round(x["app_avg"], 4),
            "seqs_per_s": round(x["S"] * world / (xms * 1e-3), 1), "partition": x["part"],
            "path": "pa_decode_shared_prefix" if x["shared"] else "pa_decode",
            "unique_kv_gbs": round(x["nbytes"]["unique_kv"] / (x["dec_avg"] * 1e-3) / 1e9, 1),
            "roofline": roofline_of(wcfg, x, peak, peak_kind),
            "gpu_launches": x["launches_per_step"] * args.steps,
            "clocks": x["clocks"],
            "config": _config_dict(wcfg, args, x["part"]),
        }
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": cfg.kv_dtype,
        "data": "synthetic",
        "config": _config_dict(cfg, args, part,
                               f"inputs larger than L2 ({r['kv_gb']:.2f} GB of K/V per step), "
                               "no flush" if r["kv_gb"] > 0.126 else
                               f"K/V ({r['kv_gb']:.3f} GB per step) may stay in L2"),
        "seqs_per_s": round(seqs_all / (ms_step * 1e-3), 1),
        "pct_of_hbm_peak": {"measured_copy": round(100 * value / world / peak, 2),
                            "spec_8000": round(100 * value / world / 8000.0, 2)},
        "decode_ms": round(r["dec_avg"], 4),
        "decode_ms_eager": round(r["dec_eager"], 4),
        "launch": r["launch"],
        "append_cow_ms": round(r["app_avg"], 4),
        "unique_kv_gbs": round(nbytes["unique_kv"] / (r["dec_avg"] * 1e-3) / 1e9, 1),
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": None if e2e is None else {
            "value": round(e2e["value"], 2), "unit": "GB/s",
            "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
            "ms_per_step": round(e2e["ms"], 4)},
        "gpu_launches": r["launches_per_step"] * args.steps,
        "clocks": r["clocks"],
    }
    if workloads:
        line["workloads"] = workloads
    print(json.dumps(line), flush=True)


def run_e2e(args, cfg, pa, dev, part, keep_state=False):
    """Host pool + pinned host buffers + H2D / step / D2H every step, pipelined
    the way a serving loop runs: the host builds step i + 1's slots and tables
    while the GPU runs step i; every step's inputs still cross H2D and its
    output D2H inside the timed region.  keep_state: also return the last
    step's host-side inputs and output and the caches after it (for a check
    of the loop's result)."""
    g = torch.Generator().manual_seed(args.seed + 77)
    inp = wl.make_decode_inputs(cfg, seed=args.seed + 5, device=dev)
    max_ctx = inp.max_ctx + args.warmup + args.steps + 2     # sequences grow one token a step
    S, Hq, D = inp.q.shape
    bs = cfg.block_size
    NB = inp.num_blocks + S * (args.warmup + args.steps + 2) // bs + S
    kc = torch.empty((NB,) + tuple(inp.key_cache.shape[1:]), dtype=inp.key_cache.dtype, device=dev)
    vc = torch.empty_like(kc)
    for t in (kc, vc):                         # finite random contents (timing only)
        t.copy_(torch.randn(t.shape, device=dev, dtype=torch.float32).to(t.dtype))
    pool = pa.BlockPool(NB, bs)
    # shuffle the free queue: take every block, give them back in a seeded order
    ids = [pool.alloc() for _ in range(NB)]
    for i in torch.randperm(NB, generator=g).tolist():
        pool.free(ids[i])
    lens = inp.context_lens.cpu().tolist()
    seqs, parents = [], []
    prefix_blocks = []
    if cfg.prefix_tokens:                      # one owner writes the shared prefix once
        owner = pool.seq_new()
        for _ in range(cfg.prefix_tokens):
            pool.seq_append(owner)
        prefix_blocks = pool.build_block_tables([owner], cfg.prefix_tokens // bs)[0][0].tolist()
    for s in range(S):
        sid = pool.seq_new()
        have = 0
        if prefix_blocks:
            pool.seq_share_prefix(sid, prefix_blocks, cfg.prefix_tokens)
            have = cfg.prefix_tokens
        for _ in range(lens[s] - 1 - have):
            pool.seq_append(sid)
        if cfg.cow_last_block:                 # a sampling parent keeps the last block shared
            parents.append(pool.seq_fork(sid))
        seqs.append(sid)
    MB = (max(lens) + args.warmup + args.steps + 2 + bs - 1) // bs
    seq_ids = torch.tensor(seqs, dtype=torch.int64)
    # every per-step input lives in one pinned staging buffer (the model would
    # write q, k, v there; the pool writes slots, tables and lengths there), so
    # one H2D copy moves a step's inputs; one D2H copy returns its output
    parts = [("q", inp.q), ("k", inp.key_new), ("v", inp.value_new),
             ("slots", torch.empty(S, dtype=torch.int64)),
             ("tables", torch.empty((S, MB), dtype=torch.int32)),
             ("lens", torch.empty(S, dtype=torch.int32))]
    offs, total = {}, 0
    for name, t in parts:
        offs[name] = total
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    # two staging slots: the host fills step i + 1's slot (pool appends, tables)
    # while the GPU still runs step i; copy streams move inputs in and outputs
    # out beside the compute stream
    NSLOT = 2
    stage_h = [torch.empty(total, dtype=torch.uint8, pin_memory=True) for _ in range(NSLOT)]
    stage_d = [torch.empty(total, dtype=torch.uint8, device=dev) for _ in range(NSLOT)]

    def view(buf, name, like):
        nbytes = like.numel() * like.element_size()
        return buf[offs[name]:offs[name] + nbytes].view(like.dtype).view(like.shape)

    hv = [{name: view(stage_h[k], name, t) for name, t in parts} for k in range(NSLOT)]
    dv = [{name: view(stage_d[k], name, t) for name, t in parts} for k in range(NSLOT)]
    for k in range(NSLOT):
        hv[k]["q"].copy_(inp.q.cpu())
        hv[k]["k"].copy_(inp.key_new.cpu())
        hv[k]["v"].copy_(inp.value_new.cpu())
    out_h = [torch.empty(inp.q.shape, dtype=inp.q.dtype, pin_memory=True) for _ in range(NSLOT)]
    out_d = [torch.empty_like(inp.q) for _ in range(NSLOT)]
    cow_buf = torch.empty((S, 2), dtype=torch.int32)
    shared = bool(cfg.prefix_tokens) and not args.no_shared_prefix
    if shared:      # every table starts with the owner's prefix blocks
        ws_bytes = pa.pa_decode_shared_prefix_workspace_size(
            S, Hq, cfg.num_kv_heads, D, bs, max_ctx, cfg.prefix_tokens, kc.dtype)
    else:
        ws_bytes = pa.pa_decode_workspace_size(S, Hq, D, max_ctx, part)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    h2d_stream = torch.cuda.Stream(device=dev)    # inputs in: never queued behind an output
    d2h_stream = torch.cuda.Stream(device=dev)    # outputs out
    inputs_in = [torch.cuda.Event() for _ in range(NSLOT)]   # slot's inputs are on the device
    kern_done = [torch.cuda.Event() for _ in range(NSLOT)]   # slot's kernels have finished
    output_out = [torch.cuda.Event() for _ in range(NSLOT)]  # slot's output is on the host
    used = [False] * NSLOT
    total_bytes = 0

    def step(i):
        k = i % NSLOT
        if used[k]:
            inputs_in[k].synchronize()         # the copy that read this host slot has finished
        pairs = pool.step(seq_ids, MB, hv[k]["slots"], cow_buf, hv[k]["tables"], hv[k]["lens"])
        with torch.cuda.stream(h2d_stream):
            if used[k]:
                h2d_stream.wait_event(kern_done[k])    # the device slot's last reader is done
            stage_d[k].copy_(stage_h[k], non_blocking=True)
            inputs_in[k].record(h2d_stream)
        stream.wait_event(inputs_in[k])
        if used[k]:
            stream.wait_event(output_out[k])   # the slot's previous output has been read out
        if pairs.numel():
            pa.pa_copy_blocks(kc, vc, pairs)
        pa.pa_reshape_and_cache(dv[k]["k"], dv[k]["v"], kc, vc, dv[k]["slots"], inp.k_scale,
                                inp.v_scale)
        if shared:
            pa.pa_decode_shared_prefix(out_d[k], dv[k]["q"], kc, vc, dv[k]["tables"],
                                       dv[k]["lens"], max_ctx, inp.scale, cfg.prefix_tokens,
                                       ws if ws_bytes else None, inp.k_scale, inp.v_scale)
        else:
            pa.pa_decode(out_d[k], dv[k]["q"], kc, vc, dv[k]["tables"], dv[k]["lens"], max_ctx,
                         inp.scale, inp.k_scale, inp.v_scale, part, ws if ws_bytes else None)
        kern_done[k].record(stream)
        with torch.cuda.stream(d2h_stream):
            d2h_stream.wait_event(kern_done[k])
            out_h[k].copy_(out_d[k], non_blocking=True)
            output_out[k].record(d2h_stream)
        used[k] = True
        nb = algorithmic_bytes(cfg, hv[k]["lens"])
        return nb["decode"] + nb["append"]

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    h2d_stream.wait_event(e0)                 # the first timed copy starts after e0
    for i in range(args.steps):
        total_bytes += step(args.warmup + i)
    e1.record(d2h_stream)                     # after the last step's output reached the host
    e1.synchronize()
    ms = e0.elapsed_time(e1)
    assert pa.pa_device_status() == 0
    h2d = total
    d2h = out_h[0].numel() * out_h[0].element_size()
    pool.close()
    res = {"ms": ms / args.steps, "bytes": total_bytes / args.steps,
           "value": (total_bytes / args.steps) / (ms / args.steps * 1e-3) / 1e9,
           "h2d": h2d, "d2h": d2h}
    if keep_state:
        k = (args.warmup + args.steps - 1) % NSLOT
        res["state"] = {"q": hv[k]["q"].clone(), "tables": hv[k]["tables"].clone(),
                        "lens": hv[k]["lens"].clone(), "out": out_h[k].clone(),
                        "key_cache": kc.cpu(), "value_cache": vc.cpu(),
                        "scale": inp.scale, "k_scale": inp.k_scale, "v_scale": inp.v_scale}
    return res


# ------------------------------------------------------------- prefill (next row)

PREFILL_METRIC = "paged chunked-prefill attention TFLOP/s (causal, of the bf16 tensor peak)"


def _prefill_peak(timed_ms: float):
    """Measured dense bf16 peak: the sustained figure for a loop of a second or
    more (the power cap has settled), else the burst one."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        if timed_ms >= 1000.0 and "bf16_tflops_sustained" in p:
            return float(p["bf16_tflops_sustained"]), "measured sustained"
        return float(p["bf16_tflops"]), "measured burst"
    except Exception:
        # no measured file: the pool's earlier measurement, 1.59 PFLOP/s as a
        # burst and about 1.4 once the power cap has settled
        return (1400.0, "fallback sustained") if timed_ms >= 1000.0 else (1590.0, "fallback burst")


def _prefill_config_dict(cfg: wl.PrefillConfig, args, note=None):
    d = {"workload": cfg.name, "num_seqs": cfg.num_seqs, "q_heads": cfg.num_q_heads,
         "kv_heads": cfg.num_kv_heads, "head_dim": cfg.head_dim, "block_size": cfg.block_size,
         "dtype": cfg.dtype, "new_tokens": [cfg.q_lo, cfg.q_hi], "cached_tokens":
         [cfg.ctx_lo, cfg.ctx_hi], "parallelism": f"replicas{args.gpus}"}
    if note:
        d["l2"] = note
    return d


def prefill_oracle_rate(cfg: wl.PrefillConfig, seed: int, budget_s: float) -> dict:
    """The fp64 oracle on the host cores over sampled rows of the workload."""
    import oracle  # test infrastructure: only the CPU-baseline / reference legs use it
    cores = os.cpu_count() or 1
    inp = wl.make_prefill_inputs(cfg, seed=seed)
    qs = inp.query_start.cpu().tolist()
    n = inp.context_lens.cpu().tolist()
    g = torch.Generator().manual_seed(seed)
    rows, keys, nrow = [], 0, max(cores, 8)

    def run(rs):
        t0 = time.perf_counter()
        oracle.paged_prefill(inp.q, cfg.dtype, inp.key_cache, inp.value_cache, cfg.dtype,
                             inp.block_tables, inp.context_lens, inp.query_start, inp.scale,
                             rows=rs, nthreads=cores)
        return time.perf_counter() - t0

    def keys_of(rs):
        k = 0
        for t in rs:
            s = max(i for i in range(cfg.num_seqs) if qs[i] <= t)
            k += n[s] - (qs[s + 1] - qs[s]) + (t - qs[s]) + 1
        return k

    # size the sample so that one pass takes about budget_s / 2
    probe = torch.randint(0, qs[-1], (nrow,), generator=g).tolist()
    tp = max(run(probe), 1e-3)
    nrow = int(max(1, min(qs[-1], nrow * (budget_s / 2) / tp)))
    rows = torch.randint(0, qs[-1], (nrow,), generator=g).tolist()
    keys = keys_of(rows)
    t, reps = 0.0, 0
    while reps < 1 or t < budget_s / 2:
        t += run(rows)
        reps += 1
    flops = 4 * keys * cfg.num_q_heads * cfg.head_dim
    return {"tflops": flops * reps / t / 1e12, "cores": cores, "seconds": t / reps,
            "sample": f"{nrow} random query rows of the workload (all {cfg.num_q_heads} heads, "
                      f"{keys} causal keys), fp64 oracle on {cores} threads, {reps} passes"}


def run_gpu_prefill(args, cfg: wl.PrefillConfig, rank, world, local_rank):
    import paged_kv_cache_338_b200 as pa
    if args.decode_select is not None:
        pa.pa_decode_select(args.decode_select)
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    inp = wl.make_prefill_inputs(cfg, seed=args.seed + rank, device=dev)
    out = torch.empty_like(inp.q)
    kc, vc = inp.key_cache, inp.value_cache
    maxq = inp.max_query_len
    flops = wl.prefill_flops(cfg, inp.query_start, inp.context_lens)
    kv_gb = 2 * kc.numel() * kc.element_size() / 1e9

    def step(ev=None):
        pa.pa_reshape_and_cache(inp.key_new, inp.value_new, kc, vc, inp.slot_mapping)
        if ev is not None:
            ev[0].record(stream)
        pa.pa_prefill(out, inp.q, kc, vc, inp.block_tables, inp.context_lens, inp.query_start,
                      maxq, inp.scale)
        if ev is not None:
            ev[1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert pa.pa_device_status() == 0
    dist = world > 1
    if dist:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks.mark_start()
    t0.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t1.record(stream)
    torch.cuda.synchronize()
    clocks.mark_end()
    clk = clocks.stop()
    assert pa.pa_device_status() == 0
    if dist:
        torch.distributed.barrier()
    ms = t0.elapsed_time(t1)
    k_ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
    value = whole_job_rate(flops * args.steps, ms, dev) / 1e12
    ms = max_over_ranks(ms, dev)
    ms_step = ms / args.steps
    tokens_all = sum_over_ranks(inp.num_tokens, dev)
    e2e = None if args.no_e2e else prefill_e2e(args, cfg, pa, dev)
    if e2e is not None:
        e2e["value"] = whole_job_rate(e2e["flops"], e2e["ms"], dev) / 1e12
    if rank != 0:
        return
    peak, peak_kind = _prefill_peak(ms)
    achieved = flops / (k_ms * 1e-3) / 1e12
    traffic = None                  # DRAM bytes of one pa_prefill, from the committed capture
    pj = None if args.seqs else _committed_capture(f"traffic_{cfg.name}.json")
    if pj is not None:
        traffic = pj.get("dram_bytes_per_launch")
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        r = prefill_oracle_rate(cfg, args.seed, args.cpu_budget)
        cpu = {"value": round(r["tflops"], 6), "unit": "TFLOP/s", "cores": r["cores"],
               "kind": "oracle", "sample": r["sample"]}
    line = {
        "metric": PREFILL_METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype,
        "data": "synthetic",
        "config": _prefill_config_dict(cfg, args, f"K/V cache {kv_gb:.2f} GB; re-read across "
                                                  f"query tiles, no flush"),
        "tokens_per_s": round(tokens_all / (ms_step * 1e-3), 1),
        "prefill_ms": round(k_ms, 4),
        "roofline": {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "traffic": traffic,
                     "peak_kind": peak_kind, "kernel": "pa_prefill"},
        "cpu_baseline": cpu,
        "e2e": None if e2e is None else {
            "value": round(e2e["value"], 2), "unit": "TFLOP/s",
            "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
            "ms_per_step": round(e2e["ms"], 4)},
        "gpu_launches": 2 * args.steps,
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)


def prefill_e2e(args, cfg, pa, dev):
    """Public API with host buffers: each step copies the new tokens' q, k, v,
    their slots and the tables from pinned memory, runs append + prefill and
    reads the output back.  Pipelined like the decode leg: two slots, inputs in
    on one copy stream while the previous step computes, outputs out on
    another."""
    inp = wl.make_prefill_inputs(cfg, seed=args.seed + 11, device=dev)
    names = ("q", "key_new", "value_new", "slot_mapping", "block_tables", "context_lens",
             "query_start")
    host = {k: getattr(inp, k).cpu().pin_memory() for k in names}   # one copy of the inputs
    NSLOT = 2
    devb = [{k: torch.empty_like(v, device=dev) for k, v in host.items()} for _ in range(NSLOT)]
    out_d = [torch.empty_like(inp.q) for _ in range(NSLOT)]
    out_h = [torch.empty(inp.q.shape, dtype=inp.q.dtype).pin_memory() for _ in range(NSLOT)]
    maxq = inp.max_query_len
    flops = wl.prefill_flops(cfg, inp.query_start, inp.context_lens)
    stream = torch.cuda.current_stream()
    h2d_stream, d2h_stream = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    inputs_in = [torch.cuda.Event() for _ in range(NSLOT)]
    kern_done = [torch.cuda.Event() for _ in range(NSLOT)]
    output_out = [torch.cuda.Event() for _ in range(NSLOT)]
    used = [False] * NSLOT

    def step(i):
        k = i % NSLOT
        with torch.cuda.stream(h2d_stream):
            if used[k]:
                h2d_stream.wait_event(kern_done[k])     # the slot's last reader is done
            for name in names:
                devb[k][name].copy_(host[name], non_blocking=True)
            inputs_in[k].record(h2d_stream)
        stream.wait_event(inputs_in[k])
        if used[k]:
            stream.wait_event(output_out[k])            # the slot's output has been read out
        d = devb[k]
        pa.pa_reshape_and_cache(d["key_new"], d["value_new"], inp.key_cache, inp.value_cache,
                                d["slot_mapping"])
        pa.pa_prefill(out_d[k], d["q"], inp.key_cache, inp.value_cache, d["block_tables"],
                      d["context_lens"], d["query_start"], maxq, inp.scale)
        kern_done[k].record(stream)
        with torch.cuda.stream(d2h_stream):
            d2h_stream.wait_event(kern_done[k])
            out_h[k].copy_(out_d[k], non_blocking=True)
            output_out[k].record(d2h_stream)
        used[k] = True

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    steps = max(3, min(args.steps, 50))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    h2d_stream.wait_event(e0)                 # the first timed copy starts after e0
    for i in range(steps):
        step(args.warmup + i)
    e1.record(d2h_stream)
    e1.synchronize()
    ms = e0.elapsed_time(e1) / steps
    assert pa.pa_device_status() == 0
    return {"ms": ms, "value": flops / (ms * 1e-3) / 1e12, "flops": flops,
            "h2d": sum(v.numel() * v.element_size() for v in host.values()),
            "d2h": out_h[0].numel() * out_h[0].element_size()}


def run_reference_prefill(args, cfg, rank, world):
    if rank != 0:
        return
    budget = max(1.0, 150.0 / (args.warmup + args.steps))
    r = prefill_oracle_rate(cfg, args.seed, budget)
    line = {
        "impl": "reference", "metric": PREFILL_METRIC, "value": round(r["tflops"], 6),
        "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * r["seconds"], 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _prefill_config_dict(cfg, args),
        "cpu_baseline": {"value": round(r["tflops"], 6), "unit": "TFLOP/s", "cores": r["cores"],
                         "kind": "oracle", "sample": r["sample"]},
        "e2e": {"value": round(r["tflops"], 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=3, choices=sorted(wl.CONFIGS),
                    help="decode workload by number: " + ", ".join(
                        f"{k} = {c.name}" for k, c in sorted(wl.CONFIGS.items())))
    ap.add_argument("--workload", choices=sorted(wl.DECODE_WORKLOADS),
                    help="decode workload by name (overrides --config)")
    ap.add_argument("--partition", type=int, default=-1, help="-1: workload default / heuristic")
    ap.add_argument("--seed", type=int, default=2)
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="time the eagerly launched step instead of its CUDA-graph replay")
    ap.add_argument("--seqs", type=int, default=0,
                    help="profiling only: a sub-batch of this many sequences of the workload")
    ap.add_argument("--no-shared-prefix", action="store_true",
                    help="shared-prefix workload: time pa_decode instead of pa_decode_shared_prefix")
    ap.add_argument("--decode-select", type=int, default=None,
                    help="pa_decode_select bit mask for the run (tuning; default: the library's)")
    ap.add_argument("--block-size", type=int, default=0, choices=[0, 8, 16, 32],
                    help="the workload's shape with another block size (0: its own)")
    ap.add_argument("--workloads-also", default=None,
                    help="comma-separated decode workloads also timed on the device and reported "
                         "under 'workloads' (default with the default workload: " +
                         ",".join(EXTRA_WORKLOADS) + "; '' for none)")
    ap.add_argument("--op", choices=["decode", "prefill"], default="decode",
                    help="decode: the paged decode step (default); prefill: the chunked-prefill "
                         "attention step")
    ap.add_argument("--prefill-workload", default="llama3_8b_gqa_bf16_chunked_prefill",
                    choices=sorted(wl.PREFILL_CONFIGS))
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("at least 3 warm-up steps")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.op == "prefill":
        import dataclasses
        cfg = wl.PREFILL_CONFIGS[args.prefill_workload]
        if args.seqs:
            cfg = dataclasses.replace(cfg, num_seqs=min(args.seqs, cfg.num_seqs),
                                      name=cfg.name + f"_small{args.seqs}")
    else:
        cfg = wl.DECODE_WORKLOADS[args.workload] if args.workload else wl.CONFIGS[args.config]
        default_shape = not (args.seqs or args.block_size or args.workload or args.config != 3)
        if args.seqs:
            cfg = _sample_cfg(cfg, args.seqs)
        if args.block_size and args.block_size != cfg.block_size:
            import dataclasses
            cfg = dataclasses.replace(cfg, block_size=args.block_size,
                                      name=cfg.name + f"_bs{args.block_size}")
        if args.workloads_also is None:
            args.workloads_also = ",".join(EXTRA_WORKLOADS) if default_shape else ""
    if args.impl == "reference":
        (run_reference_prefill if args.op == "prefill" else run_reference)(args, cfg, rank, world)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        (run_gpu_prefill if args.op == "prefill" else run_gpu)(args, cfg, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
