"""Benchmark of the paged decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl reference]

A step is one pass of the whole hot path over one batch: copy-on-write block
copies (when the workload has any), the cache write of each sequence's new
token, and the paged decode attention of every sequence.  Default workload:
the Llama-3-8B-shaped GQA layer (32 q / 8 kv heads, head_dim 128, bf16,
block 16, 256 sequences, lognormal lengths with median 1024 in [16, 8192]).

Metric: algorithmic HBM bytes of the step / step time (GB/s), with tokens/s
beside it.  Algorithmic bytes of a decode: every (block, kv head) tile pair
the tables reach (2 * B * D * 2 bytes each) + q + out + block-table entries +
seq_lens; of a cache write: new K/V read + written + slots; of a copy: block
bytes read + written + pairs.

Timing: W untimed steps, then K steps between barriers and device syncs,
measured with CUDA events on the launching stream (max over ranks for N>1).
Per-step K/V (1.4 GB here) is far larger than the 126 MB L2, so no flush is
needed between steps.  The decode kernel's own time comes from events around
each launch inside the timed region.  The e2e figure repeats the step through
``PagedDecodeStep`` from pinned host buffers: host->device copies of every
step's inputs and the device->host copy of every output are inside its timed
region (they overlap neighbouring steps' kernels, as in a serving loop).  N>1 runs independent sequence shards per GPU (weak scaling); the
path has no exchange step.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "paged decode-attention HBM GB/s and % of roofline; tokens/s at Llama-3-8B GQA"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0  # dense bf16 / fp16 tensor throughput (burst), when the measured one is absent
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "pa_decode_llama3_8b.md")
KERNEL_SOURCES = [
    os.path.join(ROOT, "paged_kv_cache_357_b200", "csrc", name)
    for name in ("pa_decode.cu", "pa_decode_tc.cu", "pa_decode_tc_blocks.cu", "pa_attn_tc.cuh",
                 "pa_decode_common.cuh", "pa_device.cuh")
]


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description="paged decode step benchmark")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", default="llama3_8b")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle time for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--num-ctas", type=int, default=0)
    ap.add_argument("--decode", default="plain", choices=["plain", "shared_prefix", "cuda_cores"],
                    help="shared_prefix: pa_decode_shared_prefix over the workload's prompt groups; "
                         "cuda_cores: pa_decode held to its CUDA-core kernel (PA_DECODE_CUDA_CORES_ONLY)")
    ap.add_argument("--max-group", type=int, default=4, help="members per shared-prefix group")
    ap.add_argument("--step", default="one_launch", choices=["one_launch", "separate"],
                    help="one_launch: the step's new-token writes inside the tensor-core decode's launch "
                         "(pa_decode_update and friends; block copies stay their own launch) where that kernel "
                         "runs; separate: pa_copy_blocks, pa_cache_write and the decode as their own launches")
    ap.add_argument("--batch", type=int, default=0,
                    help="sequences per GPU for the llama7b / llama3_8b(_spec4, _prefill256) / llama2_70b_shared "
                         "workloads (0 = the workload's own)")
    return ap.parse_args(argv)


# ---------------------------------------------------------------------------
# byte accounting
# ---------------------------------------------------------------------------


def step_bytes(L, mode: str = "plain") -> dict:
    """Algorithmic bytes of one step.  The decode reads every (block, kv
    head) K/V tile its sequences reference — once per sequence, or, with
    mode "shared_prefix", once per distinct block — plus q, out (q_len rows
    per sequence), the table entries and lengths."""
    import numpy as np

    es = 2
    B, D, Hq, Hkv, S = L.block_size, L.head_dim, L.num_q_heads, L.num_kv_heads, L.num_seqs
    nb = L.total_blocks_touched()
    tile_pair = 2 * B * D * es
    small = 2 * S * L.q_len * Hq * D * es + nb * 4 + S * 4
    per_seq = nb * Hkv * tile_pair + small
    exact = int(L.seq_lens.astype(np.int64).sum()) * Hkv * 2 * D * es + small
    unique = L.unique_blocks_touched() * Hkv * tile_pair + small
    decode = unique if mode == "shared_prefix" else per_seq
    T = L.num_new_tokens
    write = T * Hkv * D * es * 2 * 2 + T * 8
    n = L.copy_pairs.shape[0]
    copy = n * 2 * Hkv * B * D * es * 2 + n * 16
    return dict(decode=decode, decode_per_sequence=per_seq, decode_token_exact=exact, decode_unique_blocks=unique,
                write=write, copy=copy, step=decode + write + copy, tile_pair=tile_pair, tiles=nb * Hkv)


def decode_flops(L) -> int:
    """Multiply-add flops of the decode's two products, 2 * D each per
    (query row, visible token) pair: scores q . K and the weighted sum of V.
    Position i of a multi-query step sees seq_len - q_len + i + 1 tokens."""
    import numpy as np

    n = L.seq_lens.astype(np.int64)
    if L.q_len == 1:
        pairs = int(n.sum())
    else:
        ok = n >= L.q_len
        pairs = int((L.q_len * (n[ok] - L.q_len) + L.q_len * (L.q_len + 1) // 2).sum())
    return 4 * pairs * L.num_q_heads * L.head_dim


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def measured_tensor_peak():
    """Dense 16-bit tensor TFLOP/s for a kernel timed on its own: the
    measured burst figure, else the fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def tensor_bound(L) -> bool:
    """Workloads whose decode runs the query-major prefill kernel: bound by
    the tensor core and the exponentials, not by HBM."""
    return L.q_len > 1 and L.head_dim == 128 and L.block_size in (8, 16, 32) and L.group * L.q_len >= 128


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def decode_kernel_name(L, mode: str = "plain") -> str:
    """Which decode kernel(s) the library runs for this workload."""
    if L.q_len > 1:
        if tensor_bound(L):
            return "pa_prefill_tc_kernel, query-major 128-row tiles (tcgen05)"
        return "pa_decode_tc_kernel, multi-query (tcgen05)"
    if mode == "shared_prefix":
        return "pa_decode_tc_kernel, group units: shared prefix once, then each member's blocks (tcgen05)"
    if mode != "cuda_cores" and L.head_dim == 128 and L.block_size in (8, 16, 32) and L.group in (1, 2, 4, 8):
        return "pa_decode_tc_kernel (tcgen05)"
    return "pa_decode_kernel (CUDA cores)"


def roofline_of(L, mode, achieved_gbs, peak_gbs, peak_kind, nbytes, decode_ms, fused=False) -> dict:
    """The decode kernel's roofline: HBM bytes for the decode kernels (with
    the step's copy and write bytes when they run in the same launch); for
    the prefill kernel the algorithmic tensor arithmetic (4 D flops per
    query row and visible token) against the dense 16-bit tensor peak."""
    if tensor_bound(L):
        tpeak, tkind = measured_tensor_peak()
        tflops = decode_flops(L) / (decode_ms * 1e-3) / 1e12
        return {
            "kernel": decode_kernel_name(L, mode),
            "bound": "tensor",
            "achieved": tflops,
            "peak": tpeak,
            "peak_kind": f"{tkind} (MEASURED_PEAKS.json bf16_tflops)" if tkind == "measured" else tkind,
            "unit": "TFLOP/s",
            "frac": tflops / tpeak,
            "frac_of_2250_nominal": tflops / 2250.0,
            "traffic": None,
            "algorithmic_flops_per_launch": decode_flops(L),
            "hbm_gbs_beside": achieved_gbs,
        }
    name = decode_kernel_name(L, mode)
    if fused:
        name += ", with the step's new-token writes in the same launch"
    return {
        "kernel": name,
        "bound": "hbm",
        "achieved": achieved_gbs,
        "peak": peak_gbs,
        "peak_kind": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else peak_kind,
        "unit": "GB/s",
        "frac": achieved_gbs / peak_gbs,
        "frac_of_8000_nominal": achieved_gbs / 8000.0,
        "traffic": profiled_traffic(L, mode, fused),
        "algorithmic_bytes_per_launch": nbytes["decode"] + nbytes["write"] if fused else nbytes["decode"],
    }


# Attention layers of the model whose layer shape a workload takes (the
# models' published layer counts), for the implied per-model token rate.
MODEL_LAYERS = {"llama7b": 32, "llama3_8b": 32, "llama2_70b": 80, "opt13b": 40}


def model_layers(L):
    for prefix, n in MODEL_LAYERS.items():
        if L.name.startswith(prefix):
            return prefix, n
    return None, None


def workload_config(L, world: int, mode: str, nbytes) -> dict:
    """The workload keys of the JSON line's config, the same for both arms."""
    import numpy as np

    return {
        "workload": L.name,
        "note": L.note,
        "global_batch": L.num_seqs * world,
        "seq_len": {"mean": float(np.mean(L.seq_lens)), "min": int(L.seq_lens.min()),
                    "max": int(L.seq_lens.max())},
        "q_len": L.q_len,
        "decode": mode,
        "l2": f"no flush: per-step K/V {nbytes['decode'] / 1e9:.2f} GB > 126 MB L2",
        "parallelism": f"dp{world} (independent sequence shards, no collective)",
    }


def decode_entry(L, mode: str) -> str:
    if L.q_len > 1:
        return "pa_decode_multi"
    return "pa_decode_shared_prefix" if mode == "shared_prefix" else "pa_decode"


def one_launch_step(L, mode: str, step: str) -> bool:
    """Whether the step's new-token writes run inside the tensor-core
    decode's launch (the *_update entry points): the tensor-core decode
    family, not the prefill or CUDA-core kernels, which take the update as
    separate launches."""
    if step != "one_launch" or mode == "cuda_cores" or tensor_bound(L):
        return False
    return L.num_new_tokens > 0


def profiled_traffic(L, mode: str = "plain", fused: bool = True):
    """dram read+write bytes per launch of the default workload's one-launch
    step (cache write + decode) from the committed ncu summary, or None for
    other workloads or launch forms, when there is no summary, or when the
    kernel source changed since it was taken."""
    if L.name != "llama3_8b" or mode != "plain" or L.num_seqs != 256 or not fused:
        return None
    try:
        text = open(PROFILE_SUMMARY).read()
    except OSError:
        return None
    m_hash = re.search(r"kernel_source_sha256:\s*([0-9a-f]+)", text)
    m_traf = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not m_hash or not m_traf or m_hash.group(1) != kernel_source_hash():
        return None
    return float(m_traf.group(1))


def host_link_gbs(dev, h2d_bytes: int, d2h_bytes: int, reps: int = 20) -> dict:
    """Pinned host<->device copy bandwidth for one step's bytes, each
    direction alone, CUDA events on a side stream."""
    import torch

    out = {}
    stream = torch.cuda.Stream(device=dev)
    for name, nbytes, to_dev in (("h2d", h2d_bytes, True), ("d2h", d2h_bytes, False)):
        host = torch.empty(max(nbytes, 1), dtype=torch.uint8).pin_memory()
        devbuf = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            for i in range(reps + 3):
                if i == 3:
                    a.record(stream)
                if to_dev:
                    devbuf.copy_(host, non_blocking=True)
                else:
                    host.copy_(devbuf, non_blocking=True)
            b.record(stream)
        stream.synchronize()
        out[name] = nbytes * reps / (a.elapsed_time(b) * 1e-3) / 1e9
    return out


def max_over_ranks(values, device="cpu"):
    """Element-wise max of per-rank timings over the default process group
    (identity with one rank).  NCCL needs a CUDA device, gloo runs on CPU."""
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def whole_job_gbs(world: int, bytes_per_step_per_rank: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank moves its own shard's bytes in the
    slowest rank's step time (weak scaling)."""
    return world * bytes_per_step_per_rank / (ms_per_step * 1e-3) / 1e9


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100", "-i",
                 gpu_id], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def gpu_id_for(device_index: int) -> str:
    import torch

    try:
        u = str(torch.cuda.get_device_properties(device_index).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(device_index)


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline leg and the reference arm)
# ---------------------------------------------------------------------------


def oracle_sample_step(L, seqs):
    """Build a bounded sample (untimed), then time one oracle step on it."""
    import oracle
    from workloads import fill_values_numpy, restrict_layout

    R = restrict_layout(L, seqs)
    V = fill_values_numpy(R)
    t0 = time.perf_counter()
    kp, vp = V.k_pool, V.v_pool
    if R.copy_pairs.shape[0] > 0:
        kp, vp = oracle.copy_blocks(kp, vp, R.copy_pairs)
    if R.num_new_tokens > 0:
        kp, vp = oracle.cache_write(kp, vp, V.new_k, V.new_v, R.slot_mapping)
    if R.q_len > 1:
        oracle.decode_multi(V.q, kp, vp, R.block_tables, R.seq_lens, R.scale, R.num_kv_heads, R.dtype)
    else:
        oracle.decode(V.q, kp, vp, R.block_tables, R.seq_lens, R.scale, R.num_kv_heads, R.dtype)
    dt = time.perf_counter() - t0
    return dt, step_bytes(R)["step"]


def host_cores() -> dict:
    """Logical CPUs of the host and those this process may run on (nproc)."""
    total = os.cpu_count() or 1
    try:
        usable = len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        usable = total
    return {"cpu_count": total, "nproc": usable}


def _oracle_worker(args):
    """One worker of the all-cores leg: the oracle steps of its sequences,
    one at a time; returns (oracle seconds, bytes).  Runs in a spawned
    process with one BLAS thread."""
    config, batch, seqs = args
    from threadpoolctl import threadpool_limits

    L = make_layout(argparse.Namespace(config=config, batch=batch))
    t_tot, b_tot = 0.0, 0
    with threadpool_limits(1):
        for s in seqs:
            dt, nbytes = oracle_sample_step(L, [int(s)])
            t_tot += dt
            b_tot += nbytes
    return t_tot, b_tot


def _oracle_worker_ready(_):
    import numpy  # noqa: F401

    import oracle  # noqa: F401
    import workloads  # noqa: F401

    return os.getpid()


def oracle_all_cores(args, L, order, per_seq_s: float, budget_s: float, workers: int) -> dict:
    """The oracle as it stands on all usable host cores: `workers` spawned
    processes (spawned, never forked, so that no CUDA state is inherited)
    take whole sequences of the same seeded order round-robin and run at the
    same time.  The leg's time is the slowest worker's oracle time."""
    import multiprocessing as mp

    n = int(max(workers, min(L.num_seqs, budget_s * workers / max(per_seq_s, 1e-6))))
    n = min(n, L.num_seqs)
    seqs = [int(s) for s in order[:n]]
    parts = [seqs[w::workers] for w in range(workers)]
    parts = [p for p in parts if p]
    ctx = mp.get_context("spawn")
    env_before = os.environ.get("OMP_NUM_THREADS")
    os.environ["OMP_NUM_THREADS"] = "1"
    try:
        with ctx.Pool(len(parts)) as pool:
            pool.map(_oracle_worker_ready, range(len(parts)), chunksize=1)  # start-up outside the timing
            res = pool.map(_oracle_worker, [(args.config, args.batch, p) for p in parts], chunksize=1)
    finally:
        if env_before is None:
            os.environ.pop("OMP_NUM_THREADS", None)
        else:
            os.environ["OMP_NUM_THREADS"] = env_before
    t_max = max(t for t, _ in res)
    nbytes = sum(b for _, b in res)
    return {"value": nbytes / t_max / 1e9, "processes": len(parts), "sequences": n, "seconds": t_max}


def cpu_baseline(L, budget_s: float, args=None) -> dict:
    """The oracle as it stands on a bounded sample of the workload: whole
    sequences in a seeded order until ~budget_s of oracle time on one
    thread; then, with `args`, the same kind of sample on every usable host
    core (one process per core, one BLAS thread each)."""
    import numpy as np
    from threadpoolctl import threadpool_limits

    order = np.random.default_rng(0).permutation(L.num_seqs)
    t_tot, b_tot, n = 0.0, 0, 0
    with threadpool_limits(1):
        for s in order:
            dt, nbytes = oracle_sample_step(L, [int(s)])
            t_tot += dt
            b_tot += nbytes
            n += 1
            if t_tot >= budget_s:
                break
    value_1t = b_tot / t_tot / 1e9
    cores = host_cores()
    out = {"value": value_1t, "unit": "GB/s", "cores": 1, "threads": 1, "kind": "oracle",
           "host_cores": cores, "value_1t": value_1t, "value_all": None,
           "sample": f"{n} of {L.num_seqs} sequences (seeded order), all heads, full step, float64 NumPy, "
                     f"1 thread, {t_tot:.1f} s"}
    if args is not None and cores["nproc"] > 1:
        allc = oracle_all_cores(args, L, order, t_tot / n, budget_s, cores["nproc"])
        out.update(value=allc["value"], cores=allc["processes"], threads=allc["processes"],
                   value_all=allc["value"])
        out["sample"] = (f"value = all cores: {allc['sequences']} of {L.num_seqs} sequences (seeded order) "
                         f"round-robin over {allc['processes']} spawned processes of one BLAS thread, "
                         f"slowest process {allc['seconds']:.1f} s of oracle time; value_1t: "
                         + out["sample"])
    return out


def make_layout(args):
    from workloads import CONFIGS, config_llama2_70b_shared, config_llama3_8b, config_llama3_8b_prefill, config_llama7b

    if args.batch:
        def shared(batch):
            if batch % 4:
                raise SystemExit("llama2_70b_shared forks every prompt into 4 samples: --batch is a multiple of 4")
            return config_llama2_70b_shared(num_prompts=batch // 4)

        makers = {"llama3_8b": config_llama3_8b, "llama7b": config_llama7b,
                  "llama3_8b_spec4": lambda batch: config_llama3_8b(batch=batch, q_len=4),
                  "llama3_8b_prefill256": lambda batch: config_llama3_8b_prefill(batch=batch),
                  "llama2_70b_shared": shared}
        if args.config not in makers:
            raise SystemExit(f"--batch applies to {sorted(makers)} only")
        return makers[args.config](args.batch)
    return CONFIGS[args.config]()


def run_reference(args):
    """The oracle, as it stands, timed on the host cores on bounded samples."""
    import numpy as np
    from threadpoolctl import threadpool_limits

    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    L = make_layout(args)
    order = np.random.default_rng(0).permutation(L.num_seqs)
    with threadpool_limits(1):
        t_one, _ = oracle_sample_step(L, [int(order[0])])
        per_step_budget = max(0.02, 150.0 / max(1, args.steps + args.warmup))
        k = int(max(1, min(L.num_seqs, per_step_budget / max(t_one, 1e-6))))
        times, nbytes = [], 0
        for i in range(args.warmup + args.steps):
            seqs = [int(order[(i * k + j) % L.num_seqs]) for j in range(k)]
            dt, b = oracle_sample_step(L, seqs)
            if i >= args.warmup:
                times.append(dt)
                nbytes += b
    total = sum(times)
    value = nbytes / total / 1e9
    sample = f"{k} sequence(s) of {L.num_seqs} per step (seeded order), all heads, full step, float64 NumPy, 1 thread"
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * total / len(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {**workload_config(L, int(os.environ.get("WORLD_SIZE", "1")), args.decode,
                                     step_bytes(L, args.decode)),
                   "step": "the oracle's copy, write and decode of the same step (float64, host cores)"},
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "threads": 1, "kind": "oracle",
                         "host_cores": host_cores(), "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------


def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    import paged_kv_cache_357_b200 as pa
    from workloads import fill_values_torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    pa.load()
    L = make_layout(args)
    mode = args.decode
    if mode == "shared_prefix" and not L.share_groups:
        raise SystemExit("--decode shared_prefix needs a workload whose sequences share prompt blocks")
    if mode != "plain" and L.q_len > 1:
        raise SystemExit(f"--decode {mode} is a single-position decode")
    decode_flags = pa.PA_DECODE_CUDA_CORES_ONLY if mode == "cuda_cores" else 0
    V = fill_values_torch(L, dev, value_seed=L.seed + 7 * rank)
    nbytes = step_bytes(L, mode)
    tables = torch.from_numpy(L.block_tables).to(dev)
    lens = torch.from_numpy(L.seq_lens).to(dev)
    slots = torch.from_numpy(L.slot_mapping).to(dev)
    pairs = torch.from_numpy(L.copy_pairs.reshape(-1, 2)).to(dev)
    out = torch.empty_like(V.q)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    groups = None
    if L.q_len > 1:
        ws = pa.alloc_multi_workspace(L.num_seqs, L.q_len, L.num_q_heads, V.k_pool, args.num_ctas)
    elif mode == "shared_prefix":
        g_starts, g_prefix = pa.shared_prefix_groups(L.block_tables, L.seq_lens, L.block_size, args.max_group)
        groups = (torch.from_numpy(g_starts).to(dev), torch.from_numpy(g_prefix).to(dev), g_starts, g_prefix)
        ws = pa.alloc_shared_prefix_workspace(L.num_seqs, args.max_group, L.num_q_heads, V.k_pool, args.num_ctas)
    else:
        ws = pa.alloc_decode_workspace(L.num_seqs, L.num_q_heads, V.k_pool, args.num_ctas, decode_flags)
    stream = torch.cuda.Stream(device=dev)
    has_copy, has_write = L.copy_pairs.shape[0] > 0, L.num_new_tokens > 0
    fused = one_launch_step(L, mode, args.step)
    launches_per_step = 1 + int(has_copy) + (0 if fused else int(has_write))
    # the one-launch form's new tokens; its block copies (a kernel of their
    # own either way) are enqueued in prologue(), outside the per-launch timing
    upd = dict(new_k=V.new_k, new_v=V.new_v, slot_mapping=slots) if has_write else {}

    def prologue():
        if has_copy:
            pa.pa_copy_blocks(pairs, V.k_pool, V.v_pool, status, stream=stream)
        if has_write and not fused:
            pa.pa_cache_write(V.new_k, V.new_v, slots, V.k_pool, V.v_pool, status, stream=stream)

    def decode():
        if fused:  # one launch: the step's copies and writes, then the decode
            if L.q_len > 1:
                pa.pa_decode_multi_update(V.q, V.k_pool, V.v_pool, tables, lens, L.scale, out, ws, status,
                                          num_ctas=args.num_ctas, stream=stream, **upd)
            elif mode == "shared_prefix":
                pa.pa_decode_shared_prefix_update(V.q, V.k_pool, V.v_pool, tables, lens, groups[0], groups[1],
                                                  args.max_group, L.scale, out, ws, status, num_ctas=args.num_ctas,
                                                  stream=stream, **upd)
            else:
                pa.pa_decode_update(V.q, V.k_pool, V.v_pool, tables, lens, L.scale, out, ws, status,
                                    num_ctas=args.num_ctas, flags=decode_flags, stream=stream, **upd)
        elif L.q_len > 1:
            pa.pa_decode_multi(V.q, V.k_pool, V.v_pool, tables, lens, L.scale, out, ws, status,
                               num_ctas=args.num_ctas, stream=stream)
        elif mode == "shared_prefix":
            pa.pa_decode_shared_prefix(V.q, V.k_pool, V.v_pool, tables, lens, groups[0], groups[1], args.max_group,
                                       L.scale, out, ws, status, num_ctas=args.num_ctas, stream=stream)
        else:
            pa.pa_decode(V.q, V.k_pool, V.v_pool, tables, lens, L.scale, out, ws, status, num_ctas=args.num_ctas,
                         flags=decode_flags, stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            prologue()
            decode()
    torch.cuda.synchronize(dev)
    if int(status.item()) != 0:
        raise SystemExit(f"device status {int(status.item())} during warm-up")

    # Two timed loops of K steps each.  The first gives `value`: events only
    # at its ends, so consecutive launches overlap as programmatic dependent
    # launch lets them (an event between two kernels would serialise them).
    # The second times every decode launch on its own (events around it) for
    # the roofline.
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(gpu_id_for(local))
    barrier()
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        t_start.record(stream)
        for k in range(K):
            prologue()
            decode()
        t_end.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    with torch.cuda.stream(stream):
        for k in range(K):
            prologue()
            ev[k][0].record(stream)
            decode()
            ev[k][1].record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clocks = sampler.stop()
    elapsed_ms = t_start.elapsed_time(t_end)
    decode_ms = sorted(ev[k][0].elapsed_time(ev[k][1]) for k in range(K))
    decode_mean_ms = sum(decode_ms) / K
    if int(status.item()) != 0:
        raise SystemExit(f"device status {int(status.item())} in the timed region")

    # ---- end to end through the public step API, from pinned host buffers
    host = dict(
        q=V.q.cpu().pin_memory(), tables=tables.cpu().pin_memory(), lens=lens.cpu().pin_memory(),
        new_k=V.new_k.cpu().pin_memory(), new_v=V.new_v.cpu().pin_memory(), slots=slots.cpu().pin_memory(),
        pairs=pairs.cpu().pin_memory() if has_copy else None,
    )
    if groups is not None:
        host["group_starts"] = torch.from_numpy(groups[2]).pin_memory()
        host["group_prefix"] = torch.from_numpy(groups[3]).pin_memory()
    step = pa.PagedDecodeStep(V.k_pool, V.v_pool, L.num_seqs, L.num_q_heads, L.max_blocks_per_seq,
                              max_new_tokens=L.num_new_tokens, max_copy_pairs=L.copy_pairs.shape[0],
                              scale=L.scale, num_ctas=args.num_ctas, q_len=L.q_len,
                              max_group_size=args.max_group if groups is not None else 0,
                              decode_flags=decode_flags)

    # The step's inputs live in the step's pinned staging areas (one per
    # buffer set, filled once from the host tensors above: a serving loop
    # would build its batch there), so each step uploads them in one copy.
    staged = set()

    counts = (int(host["pairs"].shape[0]) if has_copy else 0, int(host["slots"].shape[0]) if has_write else 0,
              int(host["group_prefix"].shape[0]) if groups is not None else 0)

    def e2e_step():
        k = step.steps % len(step.sets)
        if k not in staged:  # a set's inputs are built in its staging block once
            v = step.staging()
            fields = [("q", host["q"]), ("block_tables", host["tables"]), ("seq_lens", host["lens"])]
            if has_write:
                fields += [("new_k", host["new_k"]), ("new_v", host["new_v"]), ("slot_mapping", host["slots"])]
            if has_copy:
                fields.append(("copy_pairs", host["pairs"]))
            if groups is not None:
                fields += [("group_starts", host["group_starts"]), ("group_prefix_blocks", host["group_prefix"])]
            for name, src in fields:
                v[name][: src.shape[0]].copy_(src)
            staged.add(k)
        return step.run_staged(*counts)

    # untimed: every buffer set's first steps (the first runs through the
    # checking wrappers, each set's next one captures its graph)
    for _ in range(max(args.warmup, len(step.sets) + 1)):
        e2e_step()
    step.synchronize()
    K2 = max(1, min(K, 500))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    # uploads start the timed region, the last download ends it
    e0.record(step.h2d_stream)
    for _ in range(K2):
        e2e_step()
    step.flush()  # the last step's download, otherwise held back for a next step
    e1.record(step.d2h_stream)
    step.synchronize()
    barrier()
    e2e_ms = e0.elapsed_time(e1) / K2
    if step.device_status() != 0:
        raise SystemExit("device status set in the e2e loop")
    link = host_link_gbs(dev, step.last_h2d_bytes, step.last_d2h_bytes)

    # ---- max over ranks
    elapsed_ms, e2e_ms, decode_mean_ms = max_over_ranks([elapsed_ms, e2e_ms, decode_mean_ms], dev)
    ms_per_step = elapsed_ms / K
    value = whole_job_gbs(world, nbytes["step"], ms_per_step)
    tokens_per_s = world * L.num_seqs * L.q_len / (ms_per_step * 1e-3)
    peak, peak_kind = measured_hbm_peak()
    achieved = (nbytes["decode"] + (nbytes["write"] if fused else 0)) / (decode_mean_ms * 1e-3) / 1e9
    result = None
    if rank == 0:
        result = {
            "metric": METRIC,
            "value": value,
            "unit": "GB/s",
            "n_gpus": world,
            "steps": K,
            "warmup": args.warmup,
            "ms_per_step": ms_per_step,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": L.dtype,
            "data": "synthetic",
            "config": {
                **workload_config(L, world, mode, nbytes),
                "step": (("pa_copy_blocks+" if has_copy else "") + decode_entry(L, mode)
                         + "_update (cache write + decode in one launch)") if fused else "+".join(
                    (["pa_copy_blocks"] if has_copy else []) + (["pa_cache_write"] if has_write else [])
                    + [decode_entry(L, mode)]),
            },
            "tokens_per_s": tokens_per_s,
            "tokens_per_s_note": ("one new token per sequence per single-layer step" if L.q_len == 1 else
                                  f"{L.q_len} query positions per sequence per single-layer step"),
            "tokens_per_s_implied_model": (tokens_per_s / model_layers(L)[1]) if model_layers(L)[1] else None,
            "tokens_per_s_implied_model_note": (
                f"implied, attention only: the single-layer step repeated for the {model_layers(L)[1]} layers of "
                f"{model_layers(L)[0]} with nothing else in the model timed" if model_layers(L)[1] else None),
            "decode_ms": decode_mean_ms,
            "decode_ms_note": (("CUDA events around each launch of the tensor-core kernel, which also runs the "
                                "step's cache update" if fused else "CUDA events around each decode launch")
                               + ", in a second timed loop of K steps; ms_per_step comes from the first loop, "
                                 "timed by events at its two ends only"),
            "decode_tflops": decode_flops(L) / (decode_mean_ms * 1e-3) / 1e12,
            "decode_ms_p50": decode_ms[K // 2],
            "bytes": nbytes,
            "roofline": roofline_of(L, mode, achieved, peak, peak_kind, nbytes, decode_mean_ms, fused),
            "e2e": {
                "value": whole_job_gbs(world, nbytes["step"], e2e_ms),
                "unit": "GB/s",
                "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": step.last_h2d_bytes,
                "d2h_bytes_per_step": step.last_d2h_bytes,
                "steps": K2,
                "how": "PagedDecodeStep from pinned staging buffers: per step one H2D copy of the packed inputs, "
                       "the step's kernels replayed as a CUDA graph, one D2H copy of the output; three buffer "
                       "sets overlap neighbouring steps' copies and kernels",
                "link_gbs": link,
                "link_note": "this box's pinned-copy bandwidth for one step's input and output bytes, "
                             "measured outside the timed region (context: e2e is bound by it when slow)",
            },
            "gpu_launches": 2 * K * launches_per_step,
            "gpu_launches_note": "both timed loops (value's and the per-launch timing's)",
            "clocks": clocks,
        }
    if world > 1:
        barrier()
        dist.destroy_process_group()
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            result["cpu_baseline"] = cpu_baseline(L, args.cpu_budget, args)
        print(json.dumps(result), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
