#!/usr/bin/env python
"""Paged decode attention throughput on B200.

One step = the whole hot path over one batch: copy_blocks (copy-on-write pairs, when the
workload has any) -> reshape_and_cache (the step's new tokens) -> pa_decode.  The default
workload is the Llama-3-8B-shaped GQA decode: 256 sequences, 32 query / 8 KV heads,
head_dim 128, block size 16, lognormal lengths (median 1024, sigma 1) clipped to
[32, 8192], bf16, shuffled physical placement, 512-token split-K partitions.

value      = decode K+V bytes (each token's K and V rows of each KV head, once) / step time
e2e        = the same bytes / time of a step whose inputs start in pinned host memory
             (H2D of q, new K/V, slots, block tables, lengths, pairs) and whose output is
             read back to the host, all through the C ABI
roofline   = pa_decode alone: algorithmic bytes (K+V + q + out + block tables + lengths)
             per call / its mean CUDA-event duration inside the timed loop, vs the
             measured HBM copy bandwidth
cpu_baseline / --impl reference = the fp64 C oracle on the host cores, on a bounded
             sample of the same workload

Multi-GPU (torchrun): every rank runs its own batch (seeded by rank) on its own GPU, no
collective on the data path ("replicas", weak scaling); the time is the max over ranks.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_kv_cache_327_b200 import workload as W  # noqa: E402

METRIC = "paged decode attention KV GB/s (% of HBM peak); seq-tokens/s, 8B-GQA decode"
KERNEL_SOURCES = ["paged_kv_cache_327_b200/csrc/pa_decode.cuh", "paged_kv_cache_327_b200/csrc/pa_ptx.cuh",
                  "paged_kv_cache_327_b200/csrc/pa_decode_tc.cuh", "paged_kv_cache_327_b200/csrc/pa_api.cu"]
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--op", choices=["step", "swap", "cache"], default="step",
                    help="step: the decode step (default); swap: swap_blocks to / from pinned host memory; "
                         "cache: reshape_and_cache and copy_blocks alone (default workload: the 70b fork step)")
    ap.add_argument("--step", choices=list(W.STEPS_70B), default=None,
                    help="70b only: 'decode' (default: one new token per sequence) or 'fork' (every sample's "
                         "whole suffix stored in the step, with all 192 copy-on-write pairs)")
    ap.add_argument("--config", default=None, choices=list(W.CONFIG_NAMES),
                    help="workload (default: 8b; 70b with --op cache)")
    ap.add_argument("--block-size", type=int, default=None)
    ap.add_argument("--num-seqs", type=int, default=None,
                    help="smaller batch of the same config (profiling; 70b: that many shared-prefix samples)")
    ap.add_argument("--uniform-lens", default=None, metavar="LO,HI",
                    help="8b only: lengths uniform in [LO, HI] instead of the lognormal mix (with --num-seqs: "
                         "e.g. 4096 sequences of 0 to 40 tokens)")
    ap.add_argument("--partition-size", type=int, default=0)
    ap.add_argument("--out-dtype", default=None, help="f32 | f16 | bf16 (default: the query dtype)")
    ap.add_argument("--kv-dtype", default=None, choices=["e4m3"],
                    help="e4m3: the same config over an FP8 KV cache (per-tensor K/V scales)")
    ap.add_argument("--qtok", type=int, default=1,
                    help="query tokens per sequence: T > 1 runs causal multi-token attention (pa_decode_multi) "
                         "over the same config, the step storing each sequence's last T tokens")
    ap.add_argument("--prefix", action="store_true",
                    help="prefix-aware decode (pa_decode_prefix): sequences sharing their first blocks read them "
                         "once; the groups come from the block tables")
    ap.add_argument("--wide-kernel", choices=["auto", "mma", "tcgen05"], default="auto",
                    help="kernel for items of more than 8 query rows per KV head (--qtok, --prefix): the warp-MMA "
                         "kernel (default) or the 5th-generation tensor-core kernel")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-paths", action="store_true",
                    help="skip the compact measurement of the other decode paths (default run at N=1 only)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target oracle time for cpu_baseline")
    ap.add_argument("--ref-seconds", type=float, default=120.0, help="target total time of --impl reference")
    args = ap.parse_args()
    if args.config is None:
        args.config = "70b" if args.op == "cache" else "8b"
    return args


def make_workload(args, seed=None, num_seqs=None):
    """The bench's workload: the config (with --block-size, --kv-dtype, --qtok, --step) and, for
    profiling, a smaller batch of it (70b: that many shared-prefix samples, in groups of 4)."""
    extra = {}
    if num_seqs:
        extra = {"num_groups": max(1, num_seqs // 4)} if args.config == "70b" else {"num_seqs": num_seqs}
    if args.qtok > 1:
        extra["num_q_tokens"] = args.qtok
    if args.step:
        if args.config != "70b":
            raise SystemExit("--step applies to the 70b config")
        extra["step"] = args.step
    if getattr(args, "uniform_lens", None):
        if args.config != "8b":
            raise SystemExit("--uniform-lens applies to the 8b config")
        lo, hi = (int(x) for x in args.uniform_lens.split(","))
        extra["uniform_lens"] = (lo, hi)
    return W.make_config(args.config, block_size=args.block_size, seed=seed, kv_dtype=args.kv_dtype, **extra)


def cpu_model() -> str:
    """The host CPU's model name (from /proc/cpuinfo), or the platform's processor string."""
    try:
        for line in open("/proc/cpuinfo", encoding="utf-8"):
            if line.lower().startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def workload_label(w: W.Workload) -> str:
    kv = w.kv_dtype if w.kv_dtype != "e4m3" else f"e4m3 (scales {w.k_scale:.4g}/{w.v_scale:.4g}, new tokens {w.new_kv_dtype})"
    qt = f", {w.num_q_tokens} query tokens per seq (causal)" if w.num_q_tokens > 1 else ""
    return (f"{w.name}: {w.num_seqs} seqs, {w.num_q_heads}/{w.num_kv_heads} heads, head_dim {w.head_dim}, "
            f"block {w.block_size}, {w.notes.get('lens', '')}, q {w.q_dtype}, kv {kv}{qt}")


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback 6.65 TB/s (no MEASURED_PEAKS.json)"


def rank_seed(config: str, rank: int) -> int:
    """Each replica decodes its own batch: the config's seed offset by the rank."""
    return W.config_seed(config) + 1000 * rank


def max_over_ranks(x: float, dist=None, device="cpu") -> float:
    """The slowest rank's value (time is taken as the max over ranks); identity without a group."""
    if dist is None:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(bytes_per_rank: int, world: int, seconds: float) -> float:
    """Whole-job GB/s: every rank processes bytes_per_rank in `seconds` (the max over ranks)."""
    return world * bytes_per_rank / seconds / 1e9


def sources_digest():
    """Digest of the kernel sources' code: // comments and blank lines are left out, so that a
    comment edit does not invalidate the recorded ncu traffic."""
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            for line in f:
                code = line.split("//", 1)[0].rstrip() if '"' not in line else line.rstrip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def wide_kernel_used(w, wide: str, max_members: int = 1):
    """The kernel the library runs for this workload's wide items (None: items of at most 8 query
    rows, which run on the decode kernel): the rule of include/pa.h's PA_OPT_WIDE_KERNEL."""
    rows = w.num_q_tokens * max_members * (w.num_q_heads // w.num_kv_heads)
    if rows <= 8:
        return None
    tc_shape = (w.head_dim == 128 and w.block_size == 16 and w.kv_dtype in ("bf16", "f16")
                and w.q_dtype == w.kv_dtype)
    if tc_shape and (wide == "tcgen05" or (wide == "auto" and rows > 32)):
        return "tcgen05"
    return "mma"


def profile_name(args, kernel=None) -> str:
    """Name of the committed ncu summary of this run's partition kernel: config, cache dtype and
    query tokens (pa_decode_partition_8b, pa_decode_partition_8b_e4m3, pa_decode_partition_8b_T5),
    with _tcgen05 when the wide items run on the tensor-core kernel (`kernel`, else the flag)."""
    kernel = kernel or getattr(args, "wide_kernel", "mma")
    return (f"pa_decode_partition_{args.config}" + (f"_{args.kv_dtype}" if args.kv_dtype else "")
            + (f"_T{args.qtok}" if args.qtok > 1 else "") + ("_fork" if getattr(args, "step", None) == "fork" else "")
            + ("_prefix" if args.prefix else "") + resized_suffix(args)
            + ("_tcgen05" if kernel == "tcgen05" else ""))


def resized_suffix(args) -> str:
    """A resized workload (sequences, lengths, block or partition size) has a summary of its own
    name, so it never takes the full-size summary's traffic."""
    lens = getattr(args, "uniform_lens", None)
    return ((f"_n{args.num_seqs}" if getattr(args, "num_seqs", None) else "")
            + (f"_u{lens.replace(',', '-')}" if lens else "")
            + (f"_bs{args.block_size}" if getattr(args, "block_size", None) else "")
            + (f"_p{args.partition_size}" if getattr(args, "partition_size", 0) else ""))


def recorded_traffic(name: str):
    """dram bytes per partition-kernel launch from the committed ncu summary `name`, if it was
    taken on the current kernel sources (otherwise None)."""
    path = os.path.join(ROOT, "profiles", f"{name}.md")
    if not os.path.exists(path):
        return None
    vals = {}
    for line in open(path, encoding="utf-8"):
        if line.startswith("traffic_bytes_per_launch:") or line.startswith("kernel_sources_sha256_16:"):
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip()
    if vals.get("kernel_sources_sha256_16") != sources_digest():
        return None
    try:
        return int(float(vals["traffic_bytes_per_launch"]))
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons every 200 ms while it runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None
        self.t_window = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.dev)], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def mark(self, t0, t1):
        self.t_window = (t0, t1)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        loaded = [r for r in rows if r[2] > 0.5 * max(x[2] for x in rows)] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[3]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(loaded)}


def oracle_post_step(w: W.Workload):
    """The cache state after the step, by the oracle's own cache operations."""
    import oracle

    kc, vc = w.k_cache.copy(), w.v_cache.copy()
    oracle.copy_blocks(kc, vc, w.copy_pairs)
    if w.kv_dtype == "e4m3":
        oracle.reshape_and_cache_e4m3(w.new_k, w.new_v, kc, vc, w.slot_mapping, w.new_kv_dtype, w.k_scale, w.v_scale)
    else:
        oracle.reshape_and_cache(w.new_k, w.new_v, kc, vc, w.slot_mapping, w.kv_dtype)
    return kc, vc


def oracle_sampler(w: W.Workload, threads: int = 0):
    """The fp64 oracle made ready to time on w (the caches after the step, and a pilot run that sizes
    the samples), on `threads` threads (0: every core the process may run on).  Returns
    sample(seconds, start) -> (KV bytes processed, seconds, threads, sequence count), which times the
    oracle on consecutive sequences (from `start`, wrapping) until ~`seconds` of work."""
    import oracle

    threads = threads or oracle.default_threads()
    kc, vc = oracle_post_step(w)
    if w.num_q_tokens > 1:
        def run(q, bt, sl, num_threads):
            return oracle.decode_multi(q, w.q_dtype, kc, vc, w.kv_dtype, bt, sl, w.scale, num_threads=num_threads)
    else:
        def run(q, bt, sl, num_threads):
            return oracle.decode(q, w.q_dtype, kc, vc, w.kv_dtype, bt, sl, w.scale, num_threads=num_threads,
                                 k_scale=w.k_scale, v_scale=w.v_scale)
    row = 2 * w.kv_row_bytes
    # pilot: one sequence of median length to size the sample
    med = int(np.argsort(w.seq_lens)[w.num_seqs // 2])
    t = time.perf_counter()
    run(np.ascontiguousarray(w.q[[med]]), np.ascontiguousarray(w.block_tables[[med]]), w.seq_lens[[med]], 1)
    per_token = (time.perf_counter() - t) / max(1, int(w.seq_lens[med]))
    # tokens per second on all threads: first the pilot's estimate, then what the last sample measured
    rate = [threads / max(per_token, 1e-12)]

    def sample(seconds: float, start: int = 0, max_len: int = 0):
        # at least one sequence per thread, so that every core has work; a sequence is one thread's
        # job, so with max_len > 0 only sequences of at most max_len tokens are taken (the pass then
        # lasts about as long as its longest sequence)
        budget_tokens = seconds * rate[0]
        pick, tok = [], 0
        for k in range(w.num_seqs):
            i = (start + k) % w.num_seqs
            if tok >= budget_tokens and len(pick) >= min(threads, w.num_seqs):
                break
            if max_len and int(w.seq_lens[i]) > max_len:
                continue
            pick.append(i)
            tok += int(w.seq_lens[i])
        if not pick:  # every sequence is longer: the shortest one
            pick = [int(np.argmin(w.seq_lens))]
            tok = int(w.seq_lens[pick[0]])
        idx = np.asarray(pick)
        q, bt, sl = (np.ascontiguousarray(w.q[idx]), np.ascontiguousarray(w.block_tables[idx]),
                     np.ascontiguousarray(w.seq_lens[idx]))
        passes, t = 0, time.perf_counter()
        while True:  # whole passes over the sample until the time budget is used
            run(q, bt, sl, threads)
            passes += 1
            dt = time.perf_counter() - t
            if dt >= 0.8 * seconds:
                break
        rate[0] = passes * tok / max(dt, 1e-9)
        return passes * tok * row, dt, threads, passes * len(idx)

    sample.per_token = per_token
    return sample


def oracle_sample_rate(w: W.Workload, seconds: float, start: int = 0, threads: int = 0):
    """One timed sample of the fp64 oracle on w (see oracle_sampler)."""
    return oracle_sampler(w, threads)(seconds, start)


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = make_workload(args)
    # the caches and the pilot once; then every step is one timed sample, sized so that the whole run
    # takes about --ref-seconds whatever --steps and --warmup are
    sample = oracle_sampler(w)
    per_step = args.ref_seconds / max(1, args.steps + args.warmup)
    # the longest sequence one thread decodes within a step's share: with many steps the sample leans
    # to the shorter sequences (the line's sample description says so), on which the oracle runs
    # faster per byte than on the whole batch
    max_len = max(int(per_step / max(sample.per_token, 1e-12)), 1)
    max_len = 0 if max_len >= int(w.seq_lens.max()) else max_len
    start = 0
    for _ in range(args.warmup):
        _, _, _, n = sample(per_step, start, max_len)
        start += n
    total_b, total_t, threads, seqs = 0, 0.0, 1, 0
    for _ in range(args.steps):
        b, t, threads, n = sample(per_step, start, max_len)
        start += n
        total_b += b
        total_t += t
        seqs += n
    value = total_b / total_t / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * total_t / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_label(w)},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "cpu_model": cpu_model(),
                         "sample": f"{seqs} sequences over {args.steps} steps (consecutive windows of the batch"
                                   + (f", sequences of at most {max_len} tokens" if max_len else "")
                                   + "), fp64 two-pass softmax, attention only"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# The other decode paths, measured after the headline step in the same run (N = 1): config, flags
PATHS = [
    ("8b_e4m3", dict(config="8b", kv_dtype="e4m3")),
    ("8b_e4m3_bs32", dict(config="8b", kv_dtype="e4m3", block_size=32)),
    ("8b_T5", dict(config="8b", qtok=5)),
    ("8b_T8", dict(config="8b", qtok=8)),
    ("8b_T16", dict(config="8b", qtok=16)),
    ("8b_T16_mma", dict(config="8b", qtok=16, wide_kernel="mma")),
    ("8b_T8_tcgen05", dict(config="8b", qtok=8, wide_kernel="tcgen05")),
    ("8b_T5_bs32", dict(config="8b", qtok=5, block_size=32)),
    ("70b_prefix", dict(config="70b", prefix=True)),
    ("70b", dict(config="70b")),
    ("7b", dict(config="7b")),
    ("13b", dict(config="13b")),
    ("13b_bs32", dict(config="13b", block_size=32)),
]


def measure_path(args, overrides: dict, calls: int = 200, warm: int = 10) -> dict:
    """One decode path (after its step's cache writes): the mean CUDA-event time of `calls`
    back-to-back decode calls (inputs larger than L2), as GB/s of algorithmic bytes (distinct
    K+V, q, out, tables) and as a fraction of the measured HBM peak."""
    from paged_kv_cache_327_b200 import binding as B

    a = argparse.Namespace(**{**vars(args), "block_size": None, "kv_dtype": None, "qtok": 1, "prefix": False,
                              "step": None, "uniform_lens": None, **overrides})
    w = make_workload(a)
    B.set_wide_kernel(a.wide_kernel)  # a path may name its own wide-item kernel
    try:
        return _measure_path(a, w, calls, warm)
    finally:
        B.set_wide_kernel(args.wide_kernel)


def _measure_path(a, w, calls, warm) -> dict:
    from paged_kv_cache_327_b200 import binding as B
    from paged_kv_cache_327_b200 import block_manager as BM

    dw = B.device_workload(w)
    ws = B.DecodeWorkspace.for_workload(dw)
    out = torch.empty(tuple(dw.q.shape), dtype=B._NAME_TORCH[w.q_dtype], device="cuda")
    B.run_step(dw, out, ws)
    if a.prefix:
        groups = torch.from_numpy(BM.find_prefix_groups(w.block_tables, w.seq_lens, w.block_size)).cuda()
        mm = B.max_prefix_members(w.num_q_heads, w.num_kv_heads)
        f = lambda: B.pa_decode_prefix(out, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, w.scale,
                                       ws.tensor, groups, mm)
    elif w.num_q_tokens > 1:
        f = lambda: B.pa_decode_multi(out, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, w.scale,
                                      ws.tensor)
    elif w.kv_dtype == "e4m3":
        f = lambda: B.pa_decode_fp8(out, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, w.scale,
                                    w.k_scale, w.v_scale, ws.tensor)
    else:
        f = lambda: B.pa_decode(out, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, w.scale, ws.tensor)
    for _ in range(warm):
        f()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(calls):
        f()
    e1.record()
    torch.cuda.synchronize()
    if B.pa_get_device_error() != B.PA_DEV_OK:
        raise RuntimeError(f"device error on path {overrides}")
    ms = e0.elapsed_time(e1) / calls
    io = w.io_bytes()
    nbytes = w.kv_bytes_unique() + io["q"] + io["block_tables"] + io["seq_lens"] + out.numel() * out.element_size()
    peak, _ = measured_peak()
    gbs = nbytes / (ms * 1e-3) / 1e9
    res = {"ms": round(ms, 5), "achieved_gbs": round(gbs, 1), "frac": round(gbs / peak, 4),
           "algorithmic_bytes": int(nbytes), "seq_tokens_per_s": round(w.total_tokens() / (ms * 1e-3), 1),
           "wide_kernel": wide_kernel_used(w, a.wide_kernel,
                                           B.max_prefix_members(w.num_q_heads, w.num_kv_heads) if a.prefix else 1)}
    del dw, ws, out
    torch.cuda.empty_cache()
    return res


def run_ours(args):
    from paged_kv_cache_327_b200 import binding as B
    from paged_kv_cache_327_b200 import build as pkg_build

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    pkg_build.build()
    torch.cuda.set_device(local)
    B.set_wide_kernel(args.wide_kernel)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    seed = rank_seed(args.config, rank)
    w = make_workload(args, seed, args.num_seqs)
    out_dtype = args.out_dtype or w.q_dtype
    dw = B.device_workload(w, f"cuda:{local}")
    ws = B.DecodeWorkspace.for_workload(dw, args.partition_size)
    out = torch.empty(tuple(dw.q.shape), dtype=B._NAME_TORCH[out_dtype], device="cuda")
    stream = torch.cuda.current_stream()
    groups_np = np.zeros((0, 3), np.int32)
    if args.prefix:
        from paged_kv_cache_327_b200 import block_manager as BM

        if w.num_q_tokens > 1 or w.kv_dtype == "e4m3":
            raise SystemExit("--prefix runs single-token decode over a 16-bit cache")
        groups_np = BM.find_prefix_groups(w.block_tables, w.seq_lens, w.block_size)
    groups = torch.from_numpy(groups_np).to(f"cuda:{local}")
    max_members = B.max_prefix_members(w.num_q_heads, w.num_kv_heads)
    wide_used = wide_kernel_used(w, args.wide_kernel, max_members if args.prefix else 1)

    kv_bytes = w.kv_bytes_logical()
    # with shared prefix blocks a physical byte is read once per sharer but fetched from HBM
    # about once (L2 hits): the roofline counts distinct physical bytes
    kv_unique = w.kv_bytes_unique()
    io = w.io_bytes()
    out_bytes = out.numel() * out.element_size()
    decode_bytes = kv_unique + io["q"] + io["block_tables"] + io["seq_lens"] + out_bytes
    launches_per_step = (1 if len(w.copy_pairs) else 0) + (1 if len(w.slot_mapping) else 0) + 3

    def step():
        if len(w.copy_pairs):
            B.pa_copy_blocks(dw.k_cache, dw.v_cache, dw.copy_pairs, stream=stream)
        if len(w.slot_mapping):
            store()
        decode()

    fp8 = w.kv_dtype == "e4m3"

    def store():
        if fp8:
            B.pa_reshape_and_cache_fp8(dw.new_k, dw.new_v, dw.k_cache, dw.v_cache, dw.slot_mapping, w.k_scale,
                                       w.v_scale, stream=stream)
        else:
            B.pa_reshape_and_cache(dw.new_k, dw.new_v, dw.k_cache, dw.v_cache, dw.slot_mapping, stream=stream)

    def decode():
        if args.prefix:
            B.pa_decode_prefix(out, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, w.scale, ws.tensor,
                               groups, max_members, args.partition_size, stream)
        elif w.num_q_tokens > 1:
            B.pa_decode_multi(out, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, w.scale, ws.tensor,
                              args.partition_size, stream)
        elif fp8:
            B.pa_decode_fp8(out, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, w.scale, w.k_scale,
                            w.v_scale, ws.tensor, args.partition_size, stream)
        else:
            B.pa_decode(out, dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, w.scale, ws.tensor,
                        args.partition_size, stream)

    # ---- warm-up (also checks the device error word once)
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if B.pa_get_device_error() != B.PA_DEV_OK:
        raise RuntimeError("device error during warm-up")

    clocks = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.5)
    # ---- timed region: K steps, events around every decode call
    ev_dec = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    wall0 = time.time()
    t_start.record(stream)
    for i in range(args.steps):
        if len(w.copy_pairs):
            B.pa_copy_blocks(dw.k_cache, dw.v_cache, dw.copy_pairs, stream=stream)
        if len(w.slot_mapping):
            store()
        ev_dec[i][0].record(stream)
        decode()
        ev_dec[i][1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    if dist:
        dist.barrier()
    elapsed_ms = t_start.elapsed_time(t_end)
    dec_ms = [a.elapsed_time(b) for a, b in ev_dec]
    if clocks:
        clocks.mark(wall0, wall1)
    elapsed_ms = max_over_ranks(elapsed_ms, dist, "cuda")
    if B.pa_get_device_error() != B.PA_DEV_OK:
        raise RuntimeError("device error during the timed region")

    # ---- e2e: every step uploads its inputs from pinned host memory and reads its result back.
    # As in a serving loop, the copies run on two copy streams and overlap the kernels of the
    # neighbouring steps: step i's upload may run during step i-1's kernels and its read-back
    # during step i+1's. Two sets of device input/output buffers alternate between steps, so a
    # set is only overwritten after the kernels that read it, and an output only after its read-back.
    pin = lambda t: t.cpu().pin_memory()
    names = ("q", "new_k", "new_v", "slot_mapping", "block_tables", "seq_lens", "copy_pairs")
    h_in = {n: pin(getattr(dw, n)) for n in names}
    h_in["groups"] = pin(groups)
    d_in = [{n: getattr(dw, n) for n in names} | {"groups": groups},
            {n: getattr(dw, n).clone() for n in names} | {"groups": groups.clone()}]
    d_out = [out, torch.empty_like(out)]
    h_out = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in h_in.values())
    d2h = h_out[0].numel() * h_out[0].element_size()
    e2e_steps = max(1, min(args.steps, 500))
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]    # upload of set s done
    ev_used = [torch.cuda.Event() for _ in range(2)]  # kernels reading set s / writing output s done
    ev_out = [torch.cuda.Event() for _ in range(2)]   # read-back of output s done

    def e2e_kernels(d, o):
        if len(w.copy_pairs):
            B.pa_copy_blocks(dw.k_cache, dw.v_cache, d["copy_pairs"], stream=stream)
        if len(w.slot_mapping):
            if fp8:
                B.pa_reshape_and_cache_fp8(d["new_k"], d["new_v"], dw.k_cache, dw.v_cache, d["slot_mapping"],
                                           w.k_scale, w.v_scale, stream=stream)
            else:
                B.pa_reshape_and_cache(d["new_k"], d["new_v"], dw.k_cache, dw.v_cache, d["slot_mapping"],
                                       stream=stream)
        a = (o, d["q"], dw.k_cache, dw.v_cache, d["block_tables"], d["seq_lens"], w.scale)
        if args.prefix:
            B.pa_decode_prefix(*a, ws.tensor, d["groups"], max_members, args.partition_size, stream)
        elif w.num_q_tokens > 1:
            B.pa_decode_multi(*a, ws.tensor, args.partition_size, stream)
        elif fp8:
            B.pa_decode_fp8(*a, w.k_scale, w.v_scale, ws.tensor, args.partition_size, stream)
        else:
            B.pa_decode(*a, ws.tensor, args.partition_size, stream)

    def e2e_run(n):
        for i in range(n):
            s = i % 2
            with torch.cuda.stream(up):
                if i >= 2:
                    up.wait_event(ev_used[s])
                for k, t in h_in.items():
                    d_in[s][k].copy_(t, non_blocking=True)
                ev_in[s].record(up)
            stream.wait_event(ev_in[s])
            if i >= 2:
                stream.wait_event(ev_out[s])
            e2e_kernels(d_in[s], d_out[s])
            ev_used[s].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(ev_used[s])
                h_out[s].copy_(d_out[s], non_blocking=True)
                ev_out[s].record(down)
        stream.wait_stream(down)

    e2e_run(3)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    up.wait_event(e0)
    e2e_run(e2e_steps)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    e2e_ms = max_over_ranks(e2e_ms, dist, "cuda")
    if not torch.equal(h_out[(e2e_steps - 1) % 2].to(out.device), d_out[(e2e_steps - 1) % 2]):
        raise RuntimeError("e2e read-back does not match the device result")

    clock_info = clocks.stop() if clocks else None

    # ---- L2-flushed decode timing (outside the timed region; a cross-check of the roofline)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    flushed = []
    for _ in range(10):
        flush.fill_(1)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        decode()
        b.record(stream)
        torch.cuda.synchronize()
        flushed.append(a.elapsed_time(b))
    del flush

    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    paths = None
    if world == 1 and not args.no_paths and args.config == "8b" and args.qtok == 1 and not args.kv_dtype \
            and not args.num_seqs and not args.block_size and not getattr(args, "uniform_lens", None):
        # the default run also measures every other decode path on the same GPU, clocks and peak
        del dw, ws
        torch.cuda.empty_cache()
        paths = {}
        for name, ov in PATHS:
            try:
                paths[name] = measure_path(args, ov)
            except torch.cuda.OutOfMemoryError as e:
                paths[name] = {"skipped": f"out of memory: {e}"[:120]}
        paths["_method"] = ("mean CUDA-event time of 200 back-to-back decode calls after 10 warm-up calls "
                            "(inputs larger than L2); frac of the same peak as roofline")

    ms_step = elapsed_ms / args.steps
    value = job_throughput(kv_bytes, world, ms_step * 1e-3)
    peak, peak_src = measured_peak()
    dec_mean = float(np.mean(dec_ms))
    achieved = decode_bytes / (dec_mean * 1e-3) / 1e9
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        b, t, threads, n = oracle_sample_rate(w, args.cpu_seconds)
        b1, t1, _, n1 = oracle_sample_rate(w, args.cpu_seconds / 3, threads=1)
        cpu = {"value": round(b / t / 1e9, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
               "single_core_gbs": round(b1 / t1 / 1e9, 5), "cpu_model": cpu_model(),
               "sample": f"{n} sequence decodes from the start of the batch of {w.num_seqs} "
                         f"({b / 1e9:.3f} GB of K+V), attention only, fp64 two-pass softmax, {t:.1f} s on "
                         f"{threads} threads; single core: {n1} sequence decodes ({b1 / 1e9:.3f} GB) in {t1:.1f} s"}
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.kv_dtype, "data": "synthetic",
        "config": {"workload": workload_label(w), "kv_bytes_per_step": kv_bytes, "kv_bytes_unique": kv_unique,
                   "seq_tokens_per_step": w.total_tokens(), "new_tokens_per_step": int(len(w.slot_mapping)),
                   "cow_pairs_per_step": int(len(w.copy_pairs)), "out_dtype": out_dtype,
                   "step": w.notes.get("step"),
                   "partition_size": args.partition_size or 512,
                   "wide_kernel": (f"{args.wide_kernel} ({wide_used})" if wide_used else None),
                   "prefix_groups": (f"{len(groups_np)} groups, {int(groups_np[:, 1].sum())} sequences, shared "
                                     f"tokens {sorted(set(int(x) for x in groups_np[:, 2]))}, max_members "
                                     f"{max_members}") if args.prefix else None,
                   "l2": f"inputs larger than L2 (K+V {kv_bytes / 1e9:.2f} GB vs 126 MB L2); no flush in the "
                         f"timed loop", "parallelism": f"replicas x{world}" if world > 1 else "1 GPU"},
        "seq_tokens_per_s": round(world * w.total_tokens() / (ms_step * 1e-3), 1),
        "query_tokens_per_s": round(world * w.num_seqs * w.num_q_tokens / (ms_step * 1e-3), 1),
        "pct_of_hbm_peak": round(100 * value / world / peak, 2),
        "e2e": {"value": round(job_throughput(kv_bytes, world, e2e_ms * 1e-3), 2), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 5),
                "copies": "every step uploads its inputs from pinned host memory and reads out back; "
                          "the copies of neighbouring steps overlap a step's kernels (two copy streams, "
                          "double-buffered device inputs and outputs)"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": recorded_traffic(profile_name(args, wide_used or "mma")),
                     "kernel": ("pa_decode_prefix" if args.prefix else
                                "pa_decode_multi" if w.num_q_tokens > 1 else "pa_decode")
                               + " call (plan + partition + merge kernels)",
                     "algorithmic_bytes_per_launch": decode_bytes, "launch_ms_mean": round(dec_mean, 5),
                     "launch_ms_l2_flushed_median": round(float(np.median(flushed)), 5),
                     "peak_source": peak_src},
        "cpu_baseline": cpu,
        "clocks": clock_info,
        "gpu_launches": launches_per_step * args.steps,
        "paths": paths,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_swap(args):
    """swap_blocks: a quarter of the config's sequences swapped out to pinned host memory and back,
    against plain bulk copies between the same kinds of memory (the host link's roofline)."""
    from paged_kv_cache_327_b200 import binding as B
    from paged_kv_cache_327_b200 import build as pkg_build

    pkg_build.build()
    w = make_workload(args)
    dw = B.device_workload(w)
    bs = w.block_size
    seqs = range(w.num_seqs // 4)
    blocks = np.asarray([int(b) for i in seqs for b in w.block_tables[i, :-(-int(w.seq_lens[i]) // bs)]], np.int32)
    n = len(blocks)
    hk = torch.empty((n,) + tuple(dw.k_cache.shape[1:]), dtype=dw.k_cache.dtype).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    out_pairs = torch.from_numpy(np.stack([blocks, np.arange(n, dtype=np.int32)], 1)).cuda()
    in_pairs = torch.from_numpy(np.stack([np.arange(n, dtype=np.int32), blocks], 1)).cuda()
    nbytes = 2 * n * w.block_bytes
    stream = torch.cuda.current_stream()

    def timed(fn, reps):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(True), torch.cuda.Event(True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps * 1e-3

    reps = max(3, min(args.steps, 50))
    t_out = timed(lambda: B.pa_swap_blocks(hk, hv, dw.k_cache, dw.v_cache, out_pairs, stream=stream), reps)
    t_in = timed(lambda: B.pa_swap_blocks(dw.k_cache, dw.v_cache, hk, hv, in_pairs, stream=stream), reps)
    assert B.pa_get_device_error() == B.PA_DEV_OK
    dbuf = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    hbuf = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    t_d2h = timed(lambda: hbuf.copy_(dbuf, non_blocking=True), reps)
    t_h2d = timed(lambda: dbuf.copy_(hbuf, non_blocking=True), reps)
    line = {
        "metric": "swap_blocks GB/s between the GPU pool and pinned host memory", "op": "swap",
        "value": round(nbytes / t_in / 1e9, 2), "unit": "GB/s", "n_gpus": 1, "steps": reps,
        "higher_is_better": True, "data": "synthetic", "dtype": w.kv_dtype,
        "config": {"workload": workload_label(w), "blocks": n, "block_bytes": w.block_bytes, "bytes_per_swap": nbytes},
        "swap_out_gbs": round(nbytes / t_out / 1e9, 2), "swap_in_gbs": round(nbytes / t_in / 1e9, 2),
        "roofline": {"bound": "host link", "unit": "GB/s",
                     "peak_d2h": round(nbytes / t_d2h / 1e9, 2), "peak_h2d": round(nbytes / t_h2d / 1e9, 2),
                     "frac_out": round(t_d2h / t_out, 4), "frac_in": round(t_h2d / t_in, 4),
                     "peak_source": "cudaMemcpyAsync of one contiguous pinned buffer of the same size, this run"},
        "gpu_launches": 2 * reps,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_cache(args):
    """reshape_and_cache and copy_blocks, each timed on its own (CUDA events around every launch,
    L2 flushed before each), against the measured HBM copy bandwidth.  Default workload: the 70b
    fork step (every sample's whole suffix stored, 192 copy-on-write pairs)."""
    from paged_kv_cache_327_b200 import binding as B
    from paged_kv_cache_327_b200 import build as pkg_build

    pkg_build.build()
    if args.config == "70b" and args.step is None:
        args.step = "fork"
    w = make_workload(args, num_seqs=args.num_seqs)
    dw = B.device_workload(w)
    stream = torch.cuda.current_stream()
    fp8 = w.kv_dtype == "e4m3"
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    peak, peak_src = measured_peak()

    def store():
        if fp8:
            B.pa_reshape_and_cache_fp8(dw.new_k, dw.new_v, dw.k_cache, dw.v_cache, dw.slot_mapping, w.k_scale,
                                       w.v_scale, stream=stream)
        else:
            B.pa_reshape_and_cache(dw.new_k, dw.new_v, dw.k_cache, dw.v_cache, dw.slot_mapping, stream=stream)

    def copy():
        B.pa_copy_blocks(dw.k_cache, dw.v_cache, dw.copy_pairs, stream=stream)

    def timed(fn, reps):
        for _ in range(max(3, args.warmup)):
            fn()
        torch.cuda.synchronize()
        flushed, back = [], []
        for _ in range(reps):
            flush.fill_(1)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            flushed.append(a.elapsed_time(b))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return float(np.median(flushed)), a.elapsed_time(b) / reps

    reps = max(5, min(args.steps, 200))
    T = int(len(w.slot_mapping))
    new_es = W.ELEM_BYTES[w.new_kv_dtype]
    # K and V rows read in their input dtype and written in the cache dtype, plus the slots
    store_bytes = T * w.num_kv_heads * w.head_dim * 2 * (new_es + W.ELEM_BYTES[w.kv_dtype]) + 8 * T
    P = int(len(w.copy_pairs))
    copy_bytes = 2 * 2 * P * w.block_bytes + 8 * P  # K and V blocks read and written, plus the pairs
    ops = {}
    # in the step's order: the copies (repeated, they read blocks no store has touched yet), then
    # the stores (repeated, idempotent), so the final state is the step's
    if P:
        med, mean = timed(copy, reps)
        ops["copy_blocks"] = {"pairs": P, "algorithmic_bytes": copy_bytes, "ms_l2_flushed_median": round(med, 5),
                              "ms_back_to_back_mean": round(mean, 5),
                              "achieved_gbs": round(copy_bytes / (med * 1e-3) / 1e9, 2),
                              "frac": round(copy_bytes / (med * 1e-3) / 1e9 / peak, 4)}
    if T:
        med, mean = timed(store, reps)
        ops["reshape_and_cache"] = {"tokens": T, "algorithmic_bytes": store_bytes, "ms_l2_flushed_median": round(med, 5),
                                    "ms_back_to_back_mean": round(mean, 5),
                                    "achieved_gbs": round(store_bytes / (med * 1e-3) / 1e9, 2),
                                    "frac": round(store_bytes / (med * 1e-3) / 1e9 / peak, 4)}
    if B.pa_get_device_error() != B.PA_DEV_OK:
        raise RuntimeError("device error in the cache operations")
    # the step's state is reproducible: check the caches against plain numpy indexing once
    if not fp8:
        kc, vc = W.apply_step_host(w)
        if not (np.array_equal(B.from_torch(dw.k_cache), kc) and np.array_equal(B.from_torch(dw.v_cache), vc)):
            raise RuntimeError("cache state after the timed cache operations differs from the expected state")
    main_op = "reshape_and_cache" if T else "copy_blocks"
    m = ops[main_op]
    line = {
        "metric": "reshape_and_cache / copy_blocks GB/s (% of HBM peak)", "op": "cache",
        "value": m["achieved_gbs"], "unit": "GB/s", "n_gpus": 1, "steps": reps, "warmup": max(3, args.warmup),
        "higher_is_better": True, "data": "synthetic", "dtype": w.kv_dtype,
        "config": {"workload": workload_label(w), "step": w.notes.get("step"),
                   "l2": "256 MB written before every timed launch"},
        "ops": ops,
        "roofline": {"bound": "hbm", "kernel": main_op, "achieved": m["achieved_gbs"], "peak": peak, "unit": "GB/s",
                     "frac": m["frac"],
                     "traffic": recorded_traffic(f"pa_{main_op}_{args.config}" + (f"_{args.kv_dtype}" if fp8 else "")
                                                 + (f"_{args.step}" if args.step else "") + resized_suffix(args)),
                     "peak_source": peak_src},
        "gpu_launches": 2 * reps * len(ops),
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.op == "swap":
        return run_swap(args)
    if args.op == "cache":
        return run_cache(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
