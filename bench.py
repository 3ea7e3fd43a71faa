#!/usr/bin/env python
"""Benchmark of the fused Q/K RMSNorm + RoPE hot path on B200.

One step = one call of the 3D entry point (across-heads RMSNorm + 3D RoPE +
V copy, FP8 E4M3 out) over one batch of the largest workload, the FP8 NeoX
video geometry: packed bf16 QKV [2, 29760, (24+24+24)*128], patch grid
31x24x40, channels 32/48/48, NeoX pairs, E4M3 outputs with scales 0.5 / 0.25.
Inputs are seeded synthetic tensors resident in HBM; the 1.1 GB input exceeds
the 126 MB L2, so no flush is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  (NAME: a 3D workload such as video3d, or table_hs / table_il / table_hs_f16 /
  table_d72 for the table form, timed over rotated input sets since one set
  fits in L2, or ucpe for the UCPE camera prep)
  python bench.py --impl reference ...   # the fp64 CPU oracle, bounded sample
  python bench.py --host-sweep           # host cost per call against device
                                         # time, 64 to 8192 tokens (C ABI)

Under torchrun each rank processes its own batch (weak scaling, no
collective on the data path); rank 0 prints one JSON line.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "tokens/s and achieved HBM GB/s (% of B200 peak) for fused QK-norm+RoPE, 1 GPU"
FALLBACK_HBM_GBS = 6650.0

# dram__bytes_read.sum + dram__bytes_write.sum of one launch, from the ncu
# captures summarised in profiles/ (rope3d_video3d.md, rope3d_fp8neox.md,
# rope_table.md, ucpe_cam_prep.md), valid only for the kernel sources whose
# hash is stored beside it (the bench reports null otherwise).
TRAFFIC = {
    "video3d": (377567232 + 326036992, "789f04d7c18eb74c"),
    "fp8neox": (1097157376 + 513794304, "789f04d7c18eb74c"),
    "fp8neox_nonorm": (1097140480 + 516132352, "789f04d7c18eb74c"),
    "gqa3d": (188861952 + 130926080, "789f04d7c18eb74c"),
    "table_hs": (43556096 + 1905920, "e27ddf1ef866f0f6"),
    "table_il": (25730304 + 0, "e27ddf1ef866f0f6"),
    "table_hs_f16": (42768896 + 1988608, "e27ddf1ef866f0f6"),
    "table_d72": (24805632 + 768, "e27ddf1ef866f0f6"),
    "ucpe": (263120896 + 205809920, "3edf98a9ef178c04"),
}
KERNEL_FILES = {"3d": ("rope3d.cu",), "table": ("rope_table.cu",),
                "ucpe": ("ucpe_launch.h", "ucpe.cu")}


def kernel_source_hash(form: str = "3d") -> str:
    """Hash of the code the form's kernels are built from: comments and
    whitespace are left out, so that only a change to the code itself
    invalidates the recorded traffic."""
    import re

    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "qk_rmsnorm_rope_qknr_b200", "csrc")
    for f in ("common.cuh", "launch.h", "launch_cache.h") + KERNEL_FILES[form]:
        with open(os.path.join(csrc, f)) as fh:
            code = fh.read()
        code = re.sub(r"/\*.*?\*/", " ", code, flags=re.S)
        code = re.sub(r"//[^\n]*", " ", code)
        h.update(f.encode() + " ".join(code.split()).encode())
    return h.hexdigest()[:16]


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,"
              "clocks.mem")

    def __init__(self, gpu_index: int):
        # nvidia-smi numbers GPUs physically; under CUDA_VISIBLE_DEVICES the
        # CUDA ordinal can differ, so name the GPU by its UUID when torch has it.
        self.gpu = str(gpu_index)
        try:
            import torch

            self.gpu = f"GPU-{torch.cuda.get_device_properties(gpu_index).uuid}"
        except Exception:  # noqa: BLE001 - fall back to the ordinal
            pass
        self.proc = None
        self.lines = []
        self.t = None
        self.load_from = self.load_to = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.perf_counter(), line.strip()))

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.t.join(timeout=2)

    def summary(self):
        """Median SM clock and the throttle reasons seen while the GPU was
        under load: from the start of the spin-up to the end of the timed
        region (samples of the idle start-up are left out)."""
        sm, smax, mem, reasons = [], None, [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for t, ln in self.lines:
            if self.load_from is not None and t < self.load_from:
                continue
            if self.load_to is not None and t > self.load_to + 0.15:
                continue
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
            try:
                mem.append(float(parts[9]))
            except (IndexError, ValueError):
                pass
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0,
                    "gpu": self.gpu}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax,
                "mem_mhz": statistics.median(mem) if mem else None,
                "reasons": sorted(reasons), "samples": len(sm), "gpu": self.gpu}


def host_cost_exe():
    """tests/host_cost.c built against the in-tree libqknr.so (gcc, once)."""
    pkg = os.path.join(ROOT, "qk_rmsnorm_rope_qknr_b200")
    src = os.path.join(ROOT, "tests", "host_cost.c")
    exe = os.path.join(pkg, "_build", "host_cost")
    lib = os.path.join(pkg, "libqknr.so")
    if os.path.exists(exe) and os.path.getmtime(exe) >= max(os.path.getmtime(src),
                                                             os.path.getmtime(lib)):
        return exe
    os.makedirs(os.path.dirname(exe), exist_ok=True)
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    subprocess.run(["gcc", "-O2", src, "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(cuda, "include"), "-L", pkg, "-lqknr",
                    "-L", os.path.join(cuda, "lib64"), "-lcudart", f"-Wl,-rpath,{pkg}",
                    f"-Wl,-rpath,{os.path.join(cuda, 'lib64')}", "-o", exe], check=True)
    return exe


def host_cost(form: str, tokens: int, calls: int = 200):
    """One run of the C host-cost program: host, device and wall us per call."""
    r = subprocess.run([host_cost_exe(), form, str(tokens), str(calls)], capture_output=True,
                       text=True, timeout=300)
    if r.returncode != 0:
        raise RuntimeError(f"host_cost {form} {tokens}: {r.stderr.strip()}")
    return json.loads(r.stdout.strip().splitlines()[-1])


def python_call_us(call, n: int = 200) -> float:
    """Host us per call of a Python binding call queued back to back (no sync)."""
    import torch

    for _ in range(10):
        call()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(n):
        call()
    us = (time.perf_counter() - t0) * 1e6 / n
    torch.cuda.synchronize()
    return us


def run_host_sweep(args):
    """Host cost against device time per call of both contract entry points
    from C, 64 to 8192 tokens: below the crossover (the first size whose
    device time reaches its host time) back-to-back calls leave the GPU
    waiting on the host."""
    rows = {}
    for form in ("3d", "table"):
        rows[form] = [host_cost(form, t) for t in (64, 128, 256, 512, 1024, 2048, 4096, 8192)]
    cross = {f: next((r["tokens"] for r in v if r["device_us_per_call"] >= r["host_us_per_call"]),
                     None) for f, v in rows.items()}
    # The same 3D calls through the Python binding: the wrapper and a prepared call.
    import torch

    import qk_rmsnorm_rope_qknr_b200 as Q
    import workloads as W

    w = W.WORKLOADS["fp8neox"]
    prm = dict(w.params(), pos_offset=0)
    prepared = Q.Rope3DCall(**prm)
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream
    row = (w.hq + w.hk + w.hv) * w.head_dim
    for r in rows["3d"]:
        T = r["tokens"]
        qkv = torch.zeros(T, row, dtype=torch.bfloat16, device="cuda")
        qw = torch.ones(w.hq * w.head_dim, dtype=torch.bfloat16, device="cuda")
        kw = torch.ones(w.hk * w.head_dim, dtype=torch.bfloat16, device="cuda")
        outs = [torch.empty(T, h, w.head_dim, dtype=torch.float8_e4m3fn, device="cuda")
                for h in (w.hq, w.hk, w.hv)]
        r["python_wrapper_us_per_call"] = python_call_us(
            lambda: Q.qknr_rope_3d(qkv, qw, kw, *outs, stream=stream, **prm))
        r["python_prepared_us_per_call"] = python_call_us(
            lambda: prepared(qkv, qw, kw, *outs, stream=sh))
    tcall = Q.RopeTableCall(heads_q=32, heads_k=8, head_dim=128, eps=1e-6, rotary_dim=96)
    for r in rows["table"]:
        T = r["tokens"]
        q = torch.zeros(T, 32, 128, dtype=torch.bfloat16, device="cuda")
        k = torch.zeros(T, 8, 128, dtype=torch.bfloat16, device="cuda")
        qo, ko = torch.empty_like(q), torch.empty_like(k)
        wt = torch.ones(128, dtype=torch.bfloat16, device="cuda")
        tbl = torch.zeros(T, 96, dtype=torch.float32, device="cuda")
        r["python_wrapper_us_per_call"] = python_call_us(
            lambda: Q.qknr_rope_table(q, k, qo, ko, wt, wt, tbl, eps=1e-6, rotary_dim=96,
                                      stream=stream))
        r["python_prepared_us_per_call"] = python_call_us(
            lambda: tcall(q, k, qo, ko, wt, wt, tbl, stream=sh))
    for form in ("3d", "table"):
        for key in ("python_wrapper_us_per_call", "python_prepared_us_per_call"):
            cross[form + "_" + key.replace("_us_per_call", "")] = next(
                (r["tokens"] for r in rows[form] if r["device_us_per_call"] >= r[key]), None)
    print(json.dumps({"host_sweep": rows, "crossover_tokens": cross,
                      "shapes": {"3d": "24+24+24 heads of 128, E4M3 out (fp8neox per token)",
                                 "table": "32+8 heads of 128, rotary_dim 96, fp32 table "
                                          "(table_hs per token)"}}), flush=True)
    return 0


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


# --------------------------------------------------------------- oracle arm --
def oracle_sample(w, inp_cpu, budget_s: float, chunk: int = 256):
    """Time the fp64 oracle on consecutive token chunks of the workload,
    cycling through it, until budget_s of CPU work is spent; returns (tokens
    processed, seconds, threads)."""
    import oracle as O
    from tests._util import t2u16

    if w.form == "ucpe":
        return oracle_sample_ucpe(w, inp_cpu, budget_s, chunk)
    if w.form != "3d":
        return oracle_sample_table(w, inp_cpu, budget_s, chunk)
    qkv = inp_cpu["qkv"].reshape(-1, inp_cpu["qkv"].shape[-1])
    qw, kw = t2u16(inp_cpu["q_weight"]), t2u16(inp_cpu["k_weight"])
    p = w.params()
    done, spent = 0, 0.0
    T = qkv.shape[0]
    while spent < budget_s and T > 0:
        s0 = done % T
        n = min(chunk, T - s0)
        bits = t2u16(qkv[s0:s0 + n])
        t0 = time.perf_counter()
        O.rope_3d(bits, qw, kw, pos_offset=s0, **p)
        spent += time.perf_counter() - t0
        done += n
    return done, spent, O.threads()


def oracle_sample_table(w, inp_cpu, budget_s: float, chunk: int):
    import oracle as O
    from tests._util import t2u16

    q, k, tbl = inp_cpu["q"], inp_cpu["k"], inp_cpu["rope_table"]
    qw, kw = t2u16(inp_cpu["q_weight"]), t2u16(inp_cpu["k_weight"])
    done, spent = 0, 0.0
    T = q.shape[0]
    while spent < budget_s and T > 0:
        s0 = done % T
        n = min(chunk, T - s0)
        tb = tbl[s0:s0 + n]
        tb = tb.numpy() if tb.dtype.is_floating_point and tb.element_size() == 4 else t2u16(tb)
        qb, kb = t2u16(q[s0:s0 + n]), t2u16(k[s0:s0 + n])
        t0 = time.perf_counter()
        O.rope_table(qb, kb, qw, kw, tb, w.eps, w.rotary_dim, interleaved=w.interleaved,
                     act=w.act)
        spent += time.perf_counter() - t0
        done += n
    return done, spent, O.threads()


def oracle_sample_ucpe(w, inp_cpu, budget_s: float, chunk: int):
    """The camera prep's oracle on consecutive token chunks (every head of each
    token, each batch element in turn), cycling through the workload."""
    import oracle as O
    from tests._util import t2u16

    done, spent = 0, 0.0
    B, N = w.batch, w.seq
    while spent < budget_s and B * N > 0:
        pos = done % (B * N)
        b, s0 = pos // N, pos % N
        n = min(chunk, N - s0)
        sl = slice(s0, s0 + n)
        args = (t2u16(inp_cpu["q_normed"][b:b + 1, sl]), t2u16(inp_cpu["k_normed"][b:b + 1, sl]),
                t2u16(inp_cpu["v_raw"][b:b + 1, sl]), inp_cpu["proj_q"][b:b + 1, sl].numpy(),
                inp_cpu["proj_kv"][b:b + 1, sl].numpy(), inp_cpu["rope_cos"][sl].numpy(),
                inp_cpu["rope_sin"][sl].numpy(), w.k_scale)
        t0 = time.perf_counter()
        O.ucpe_cam_prep(*args, act=w.act)
        spent += time.perf_counter() - t0
        done += n
    return done, spent, O.threads()


def one_core(w, inp_cpu, budget_s: float, chunk: int):
    """The oracle on one host thread, for the single-core figure beside the
    all-core one; returns tokens/s."""
    import oracle as O

    before = O.threads()
    O.set_threads(1)
    try:
        n, sec, _ = oracle_sample(w, inp_cpu, budget_s, chunk)
    finally:
        O.set_threads(before)
    return n / sec


def run_reference(args, w):
    """--impl reference: the oracle as it stands, on the host cores."""
    import workloads as W

    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    inp = W.make_inputs(w, device="cpu")
    # About a minute of oracle work over the whole run (6 x --cpu-seconds),
    # whatever K and W are; a step does at least one chunk, so small per-step
    # budgets use small ones.
    per_step = 6.0 * args.cpu_seconds / max(1, args.steps + args.warmup)
    chunk = 256 if per_step >= 0.5 else 32
    for _ in range(args.warmup):
        oracle_sample(w, inp, per_step, chunk)
    toks, secs = 0, 0.0
    threads = 1
    for _ in range(args.steps):
        n, s, threads = oracle_sample(w, inp, per_step, chunk)
        toks += n
        secs += s
    value = toks / secs
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "tokens": w.tokens,
                   "sample": "token chunks in order, cycling through the workload"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"{toks // max(1, args.steps)} tokens per step of {w.name} "
                                   f"(in order from its first token, cycling through its "
                                   f"{w.tokens}; {secs / max(1, args.steps):.3f} s of oracle work per step)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU arm --
def init_gpu():
    """This rank's device, and an NCCL group when launched with several ranks."""
    import torch

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))
        pg = dist
    return rank, world, local, dev, pg


def time_steps(step, args, stream, local, dev, pg):
    """A spin-up, W untimed steps, then K back-to-back steps (one kernel launch
    each, nothing else on the stream) between two events on the launching
    stream. The kernels are programmatic dependent launches, so no event may
    sit between them: the average launch duration is the region's time over K.

    The spin-up (--spin-ms, 1000 ms by default; 0 turns it off) runs untimed
    steps for that long with the clock sampler already running, so that the
    K timed steps measure the state the GPU holds under sustained load, which
    is how the op runs inside a model. On most B200 boxes that state differs
    from a cool start in two ways: the 1 kW power cap lowers the SM clock (to
    about 1560-1870 MHz for these kernels, sw_power_cap active), and the
    kernels nevertheless run faster than in the first milliseconds after idle
    (the FP8 3D workload: 260.6 us after 1 s of load at 1642 MHz against
    288 us in 20 cold launches at 1965 MHz on one box, memory clock at its
    maximum in both); on others the clock stays at 1965 MHz and the time with
    it. The bench line carries the sampled SM and memory clocks, the time
    normalised to the top SM clock, and the spread of single launches timed
    one by one after the region.
    Returns (ms per step, max over ranks; the clock sampler; the spread)."""
    import torch

    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        clocks.load_from = time.perf_counter()
        n = 0
        while (time.perf_counter() - clocks.load_from) * 1e3 < args.spin_ms:
            step(n)
            n += 1
            if n % 16 == 0:  # keep the queue short, so the spin-up ends on time
                torch.cuda.synchronize()
        for i in range(args.warmup):
            step(i)
        torch.cuda.synchronize()
        if pg:
            pg.barrier()
        torch.cuda.synchronize()
        t_start.record(stream)
        for i in range(args.steps):
            step(i)
        t_end.record(stream)
        torch.cuda.synchronize()
        clocks.load_to = time.perf_counter()
        # The spread: the same steps again, each between its own events (an
        # event between two launches ends their overlap, so these are single
        # launches, reported beside the headline, not in it).
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        for i, (a, b) in enumerate(ev):
            a.record(stream)
            step(i)
            b.record(stream)
        torch.cuda.synchronize()
    one = sorted(a.elapsed_time(b) * 1e3 for a, b in ev)
    spread = {"min_us": one[0], "median_us": one[len(one) // 2], "max_us": one[-1],
              "launches": len(one)} if one else None
    if pg:
        pg.barrier()
    total_ms = t_start.elapsed_time(t_end)
    if pg:
        t = torch.tensor([total_ms], device=dev)
        pg.all_reduce(t, op=pg.ReduceOp.MAX)
        total_ms = t.item()
    return total_ms / args.steps, clocks, spread


def clock_normalised(us_per_launch, clk):
    """The launch time in SM cycles at the median sampled clock, and that many
    cycles at the GPU's top clock: what the launch would take had the clock not
    dropped (the kernels here are partly issue-bound, so their time follows
    the SM clock). None without clock samples."""
    if not clk.get("sm_mhz") or not clk.get("sm_max_mhz"):
        return None
    cycles = us_per_launch * clk["sm_mhz"]
    return {"sm_cycles_per_launch": cycles, "us_at_sm_max": cycles / clk["sm_max_mhz"]}


def run_gpu(args, w):
    import torch

    import qk_rmsnorm_rope_qknr_b200 as Q
    import workloads as W

    rank, world, local, dev, pg = init_gpu()
    Q.lib()

    # Each rank: its own batch of the workload (seed offset by rank).
    inp = W.make_inputs(w, device=dev, seed=w.seed + rank)
    T = w.tokens
    odt = torch.float8_e4m3fn if w.output_fp8 else torch.bfloat16
    outs = [torch.empty(T, h, w.head_dim, dtype=odt, device=dev) for h in (w.hq, w.hk, w.hv)]
    p = w.params()
    if getattr(args, "tokens", None):
        p["pos_offset"] = 0  # a sequence shard of the workload: any token count
    qkv, qw, kw = inp["qkv"], inp["q_weight"], inp["k_weight"]
    stream = torch.cuda.current_stream(dev)

    def step(i):
        Q.qknr_rope_3d(qkv, qw, kw, *outs, stream=stream, **p)

    ms_per_step, clocks, spread = time_steps(step, args, stream, local, dev, pg)
    avg_launch_ms = ms_per_step
    tokens_per_s = world * T / (ms_per_step / 1e3)

    alg_bytes = W.algorithmic_bytes(w)
    peak, peak_kind = measured_peaks()
    achieved = alg_bytes / (avg_launch_ms / 1e3) / 1e9
    tr = TRAFFIC.get(w.name)
    traffic = tr[0] if tr and tr[1] == kernel_source_hash() else None

    host_us = None
    if rank == 0 and world == 1 and not args.no_e2e:
        # host cost of one call: through the Python binding (argument checks
        # and ctypes) and from C through the ABI, with the launch
        prepared = Q.Rope3DCall(**p)
        sh = stream.cuda_stream
        host_us = {"python_binding": python_call_us(lambda: step(0)),
                   "python_prepared": python_call_us(
                       lambda: prepared(qkv, qw, kw, *outs, stream=sh))}
        if not getattr(args, "tokens", None) and w.name == "fp8neox":
            hc = host_cost("3d", T)
            host_us.update({"c_abi": hc["host_us_per_call"],
                            "c_abi_device_us": hc["device_us_per_call"]})

    # End to end through the C ABI with host buffers: copy the step's input
    # from pinned host memory, run, copy the outputs back, every step.
    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(args, w, qkv, qw, kw, outs, p, stream, dev, world, pg)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        inp_cpu = {"qkv": qkv.cpu(), "q_weight": qw.cpu(), "k_weight": kw.cpu()}
        n, s, threads = oracle_sample(w, inp_cpu, args.cpu_seconds)
        cpu = {"value": n / s, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": f"{n} tokens of {w.name} in order, cycling through its {T} "
                         f"({s:.1f} s of fp64 oracle work)",
               "value_1core": one_core(w, inp_cpu, args.cpu_seconds / 4, 256)}

    if rank == 0:
        clk = clocks.summary()
        line = {
            "metric": METRIC, "value": tokens_per_s, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic",
            "config": {"workload": w.name, "tokens_per_gpu": T,
                       "io": "bf16 in, " + ("e4m3 out" if w.output_fp8 else "bf16 out"),
                       "qkv_shape": list(qkv.shape), "grid": [w.ppf, w.pph, w.ppw],
                       "channels": [w.cf, w.ch, w.cw], "heads": [w.hq, w.hk, w.hv],
                       "head_dim": w.head_dim, "interleave": w.interleave,
                       "is_qk_norm": w.is_qk_norm, "output_fp8": w.output_fp8,
                       "parallelism": f"dp{world}" if world > 1 else "single",
                       "l2": f"no flush: inputs {qkv.numel() * 2 / 1e6:.0f} MB > 126 MB L2",
                       "spin_up_ms": args.spin_ms},
            "hbm_gbs": achieved, "hbm_pct_of_peak": 100.0 * achieved / peak,
            "kernel_us": avg_launch_ms * 1e3,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "peak_source": f"{peak_kind} hbm_gbs",
                         "algorithmic_bytes_per_launch": alg_bytes},
            "cpu_baseline": cpu, "clocks": clk, "e2e": e2e, "gpu_launches": args.steps,
            "clock_normalised": clock_normalised(avg_launch_ms * 1e3, clk),
            "launch_spread": spread,
            "host_us_per_call": host_us,
        }
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    return 0


def run_gpu_table(args, w):
    """The table form (per-head norm + cos/sin table): one launch of
    qknr_rope_table per step. Its inputs are smaller than L2, so the steps
    rotate through enough input/output sets to pass 600 MB, each set evicted
    from L2 before it comes round again."""
    import torch

    import qk_rmsnorm_rope_qknr_b200 as Q
    import workloads as W

    rank, world, local, dev, pg = init_gpu()
    Q.lib()
    T = w.tokens
    alg_bytes = W.algorithmic_bytes(w)
    nsets = max(3, -(-600_000_000 // alg_bytes))
    sets = []
    for k in range(nsets):
        inp = W.make_inputs(w, device=dev, seed=w.seed + 1000 * rank + k)
        inp["q_out"], inp["k_out"] = torch.empty_like(inp["q"]), torch.empty_like(inp["k"])
        sets.append(inp)
    stream = torch.cuda.current_stream(dev)

    def run(s, st=stream):
        Q.qknr_rope_table(s["q"], s["k"], s["q_out"], s["k_out"], s["q_weight"], s["k_weight"],
                          s["rope_table"], eps=w.eps, rotary_dim=w.rotary_dim,
                          interleaved=w.interleaved, stream=st)

    # One launch moves 50-85 MB in 13-22 us, less time than the Python call
    # that issues it, so back-to-back calls would time the host. The steps are
    # therefore replayed from CUDA graphs captured once outside the timed
    # region: `full` holds one launch per rotating set, `rest` the first
    # K mod nsets; the timed region replays full K // nsets times, then rest:
    # exactly K launches.
    def capture(n):
        if n == 0:
            return None
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for k in range(n):
                run(sets[k], st=None)
        return g

    for i in range(args.warmup):
        run(sets[i % nsets])
    torch.cuda.synchronize()
    full, rest = capture(nsets), capture(args.steps % nsets)
    for g in (full, rest):
        if g is not None:
            g.replay()
    torch.cuda.synchronize()

    def region(_):
        for _ in range(args.steps // nsets):
            full.replay()
        if rest is not None:
            rest.replay()

    graph_args = argparse.Namespace(steps=1, warmup=0, spin_ms=args.spin_ms)
    ms_region, clocks, _ = time_steps(region, graph_args, stream, local, dev, pg)
    ms_per_step = ms_region / args.steps
    tokens_per_s = world * T / (ms_per_step / 1e3)
    peak, peak_kind = measured_peaks()
    achieved = alg_bytes / (ms_per_step / 1e3) / 1e9
    tr = TRAFFIC.get(w.name)
    traffic = tr[0] if tr and tr[1] == kernel_source_hash("table") else None

    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e_table(args, w, sets[0], run, stream, dev, world, pg)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        inp_cpu = {k: v.cpu() for k, v in sets[0].items() if k not in ("q_out", "k_out")}
        n, sec, threads = oracle_sample(w, inp_cpu, args.cpu_seconds, chunk=128)
        cpu = {"value": n / sec, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": f"{n} tokens of {w.name} in order, cycling through its {T} "
                         f"({sec:.1f} s of fp64 oracle work)",
               "value_1core": one_core(w, inp_cpu, args.cpu_seconds / 4, 128)}
    if rank == 0:
        clk = clocks.summary()
        q = sets[0]["q"]
        line = {
            "metric": METRIC, "value": tokens_per_s, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic",
            "config": {"workload": w.name, "tokens_per_gpu": T, "io": f"{w.act} in and out",
                       "q_shape": list(q.shape),
                       "k_shape": list(sets[0]["k"].shape), "rotary_dim": w.rotary_dim,
                       "interleaved": w.interleaved,
                       "table_dtype": "f32" if w.table_f32 else w.act,
                       "parallelism": f"dp{world}" if world > 1 else "single",
                       "l2": f"{nsets} rotated input/output sets "
                             f"({nsets * alg_bytes / 1e6:.0f} MB > 126 MB L2)",
                       "launch": f"CUDA graphs of {nsets} launches (one per set), replayed "
                                 f"for exactly K launches",
                       "spin_up_ms": args.spin_ms},
            "hbm_gbs": achieved, "hbm_pct_of_peak": 100.0 * achieved / peak,
            "kernel_us": ms_per_step * 1e3,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "peak_source": f"{peak_kind} hbm_gbs",
                         "algorithmic_bytes_per_launch": alg_bytes},
            "cpu_baseline": cpu, "clocks": clk, "e2e": e2e,
            "gpu_launches": args.steps, "clock_normalised": clock_normalised(ms_per_step * 1e3, clk),
        }
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    return 0


def measure_e2e_table(args, w, dset, run, stream, dev, world, pg):
    """End to end through the C ABI for the table form, inputs and outputs in
    page-locked host memory: staged (copy q, k and the table in, run, copy
    q_out and k_out back), zero-copy (the kernel reads and writes the host
    buffers across the bus), pipelined (8 token chunks on three streams) or
    across-steps (two device sets, step i's outputs leaving while step i+1's
    inputs arrive); the fastest is reported, beside the time of the copies
    alone. Every step moves all of its inputs in and its outputs back."""
    import torch

    names_in = ("q", "k", "q_weight", "k_weight", "rope_table")
    host = {n: torch.empty(dset[n].shape, dtype=dset[n].dtype).pin_memory() for n in names_in}
    for n in names_in:
        host[n].copy_(dset[n].cpu())
    for n in ("q_out", "k_out"):
        host[n] = torch.empty(dset[n].shape, dtype=dset[n].dtype).pin_memory()
    dev_set = {n: torch.empty_like(dset[n]) for n in dset}
    dev_set["q_weight"], dev_set["k_weight"] = dset["q_weight"], dset["k_weight"]
    hz = dict(host, q_weight=dset["q_weight"], k_weight=dset["k_weight"])
    steps = max(3, min(args.e2e_steps, args.steps))

    def staged():
        for n in ("q", "k", "rope_table"):
            dev_set[n].copy_(host[n], non_blocking=True)
        run(dev_set)
        for n in ("q_out", "k_out"):
            host[n].copy_(dev_set[n], non_blocking=True)

    def zero_copy():
        run(hz)

    # pipelined: 8 token chunks (each a table shard: its own rows of q, k and
    # the table) flow host -> device, through the kernel and back on three
    # streams, so both copy directions and the kernel overlap.
    from qk_rmsnorm_rope_qknr_b200 import sharding

    T = w.tokens
    chunks = [sharding.token_shard(T, 8, r) for r in range(8)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in chunks]
    ev_k = [torch.cuda.Event() for _ in chunks]

    def pipelined():
        for i, (s0, c) in enumerate(chunks):
            with torch.cuda.stream(s_in):
                for n in ("q", "k", "rope_table"):
                    dev_set[n][s0:s0 + c].copy_(host[n][s0:s0 + c], non_blocking=True)
                ev_in[i].record(s_in)
            stream.wait_event(ev_in[i])
            run({n: t[s0:s0 + c] if n not in ("q_weight", "k_weight") else t
                 for n, t in dev_set.items()})
            ev_k[i].record(stream)
            s_out.wait_event(ev_k[i])
            with torch.cuda.stream(s_out):
                for n in ("q_out", "k_out"):
                    host[n][s0:s0 + c].copy_(dev_set[n][s0:s0 + c], non_blocking=True)
        stream.wait_stream(s_out)

    def timed(step):
        for _ in range(2):
            step()
        torch.cuda.synchronize()
        if pg:
            pg.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            step()
        b.record(stream)
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / steps
        if pg:
            t = torch.tensor([ms], device=dev)
            pg.all_reduce(t, op=pg.ReduceOp.MAX)
            ms = t.item()
        return ms

    # across steps: two device sets on two copy streams, so that step i's
    # outputs go back while step i+1's inputs come in
    sets2 = [dev_set, {n: torch.empty_like(dset[n]) for n in dset}]
    sets2[1]["q_weight"], sets2[1]["k_weight"] = dset["q_weight"], dset["k_weight"]
    x_in, x_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    xe_in = [torch.cuda.Event() for _ in range(2)]
    xe_k = [torch.cuda.Event() for _ in range(2)]
    xe_out = [torch.cuda.Event() for _ in range(2)]
    for e in xe_out:
        e.record(x_out)
    xstep = [0]

    def across_steps():
        k = xstep[0] % 2
        xstep[0] += 1
        dv = sets2[k]
        with torch.cuda.stream(x_in):
            x_in.wait_event(xe_k[k])       # the kernel two steps back has read these
            for n in ("q", "k", "rope_table"):
                dv[n].copy_(host[n], non_blocking=True)
            xe_in[k].record(x_in)
        stream.wait_event(xe_in[k])
        stream.wait_event(xe_out[k])       # its outputs of two steps back have left
        run(dv)
        xe_k[k].record(stream)
        with torch.cuda.stream(x_out):
            x_out.wait_event(xe_k[k])
            for n in ("q_out", "k_out"):
                host[n].copy_(dv[n], non_blocking=True)
            xe_out[k].record(x_out)

    def timed_across():
        for _ in range(2):
            across_steps()
        torch.cuda.synchronize()
        if pg:
            pg.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            across_steps()
        stream.wait_stream(x_out)
        b.record(stream)
        torch.cuda.synchronize()
        ms_ = a.elapsed_time(b) / steps
        if pg:
            t = torch.tensor([ms_], device=dev)
            pg.all_reduce(t, op=pg.ReduceOp.MAX)
            ms_ = t.item()
        return ms_

    # The bus alone: the same bytes copied in and out at once, no kernel.
    s_copy = torch.cuda.Stream(dev)

    def copies_only():
        for n in ("q", "k", "rope_table"):
            dev_set[n].copy_(host[n], non_blocking=True)
        with torch.cuda.stream(s_copy):
            for n in ("q_out", "k_out"):
                host[n].copy_(dset[n], non_blocking=True)
        stream.wait_stream(s_copy)

    ms = {"staged": timed(staged), "zero-copy": timed(zero_copy), "pipelined": timed(pipelined),
          "across-steps": timed_across()}
    best = min(ms, key=ms.get)
    bus_ms = timed(copies_only)
    nbytes = lambda names: sum(dset[n].numel() * dset[n].element_size() for n in names)  # noqa
    return {"value": world * w.tokens / (ms[best] / 1e3), "unit": "tokens/s",
            "h2d_bytes_per_step": nbytes(("q", "k", "rope_table")),
            "d2h_bytes_per_step": nbytes(("q_out", "k_out")),
            "steps": steps, "mode": best,
            "ms_per_step": {k: round(v, 4) for k, v in ms.items()},
            "copies_only_ms_per_step": round(bus_ms, 4),
            "frac_of_copies_only": round(bus_ms / ms[best], 4)}


def measure_e2e(args, w, qkv, qw, kw, outs, p, stream, dev, world, pg):
    """End to end through the C ABI with the step's input and outputs in
    page-locked host memory. Three ways, all timed, the fastest reported:
      staged:    copy the input host -> device, run, copy the outputs back;
      zero-copy: hand the host buffers to qknr_rope_3d itself; the kernel's
                 bulk copies read the input across the bus and its stores
                 write the outputs back, both directions at once;
      pipelined: 8 token chunks, each copied in, transformed (as a sequence
                 shard with its pos_offset) and copied out on its own stream.
    Either way every step moves the whole input to the GPU and the whole
    output back."""
    import torch

    import qk_rmsnorm_rope_qknr_b200 as Q

    h_in = torch.empty(qkv.shape, dtype=qkv.dtype).pin_memory()
    h_in.copy_(qkv.cpu())
    h_out = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]
    d_in = torch.empty_like(qkv)
    steps = max(3, min(args.e2e_steps, args.steps))

    def staged():
        d_in.copy_(h_in, non_blocking=True)
        Q.qknr_rope_3d(d_in, qw, kw, *outs, stream=stream, **p)
        for h, o in zip(h_out, outs):
            h.copy_(o, non_blocking=True)

    def zero_copy():
        Q.qknr_rope_3d(h_in, qw, kw, *h_out, stream=stream, **p)

    # pipelined: token chunks (each a sequence shard with its own pos_offset)
    # flow host -> device, through the kernel, and back on three streams, so
    # both copy directions and the kernel overlap.
    from qk_rmsnorm_rope_qknr_b200 import sharding

    T = w.tokens
    flat_h, flat_d = h_in.reshape(T, -1), d_in.reshape(T, -1)
    P = w.ppf * w.pph * w.ppw
    chunks = [sharding.token_shard(T, 8, r) for r in range(8)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in chunks]
    ev_k = [torch.cuda.Event() for _ in chunks]

    def pipelined():
        for i, (s0, c) in enumerate(chunks):
            with torch.cuda.stream(s_in):
                flat_d[s0:s0 + c].copy_(flat_h[s0:s0 + c], non_blocking=True)
                ev_in[i].record(s_in)
            stream.wait_event(ev_in[i])
            Q.qknr_rope_3d(flat_d[s0:s0 + c], qw, kw, *(o[s0:s0 + c] for o in outs),
                           stream=stream, **dict(p, pos_offset=sharding.shard_pos_offset(s0, 0, P)))
            ev_k[i].record(stream)
            s_out.wait_event(ev_k[i])
            with torch.cuda.stream(s_out):
                for h, o in zip(h_out, outs):
                    h[s0:s0 + c].copy_(o[s0:s0 + c], non_blocking=True)
        stream.wait_stream(s_out)

    def timed(step):
        for _ in range(2):
            step()
        torch.cuda.synchronize()
        if pg:
            pg.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            step()
        b.record(stream)
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / steps
        if pg:
            t = torch.tensor([ms], device=dev)
            pg.all_reduce(t, op=pg.ReduceOp.MAX)
            ms = t.item()
        return ms

    # The bus alone: the same bytes copied in and out at once, no kernel.
    s_copy = torch.cuda.Stream(dev)

    def copies_only():
        d_in.copy_(h_in, non_blocking=True)
        with torch.cuda.stream(s_copy):
            for h, o in zip(h_out, outs):
                h.copy_(o, non_blocking=True)
        stream.wait_stream(s_copy)

    ms = {"staged": timed(staged), "zero-copy": timed(zero_copy), "pipelined": timed(pipelined)}
    best = min(ms, key=ms.get)
    bus_ms = timed(copies_only)
    return {"value": world * w.tokens / (ms[best] / 1e3), "unit": "tokens/s",
            "h2d_bytes_per_step": qkv.numel() * qkv.element_size(),
            "d2h_bytes_per_step": sum(o.numel() * o.element_size() for o in outs),
            "steps": steps, "mode": best,
            "ms_per_step": {k: round(v, 4) for k, v in ms.items()},
            "copies_only_ms_per_step": round(bus_ms, 4),
            "frac_of_copies_only": round(bus_ms / ms[best], 4)}


UCPE_INPUTS = ("q_normed", "k_normed", "v_raw", "proj_q", "proj_kv", "rope_cos", "rope_sin")


def run_gpu_ucpe(args, w):
    """The UCPE camera prep: one launch of qknr_ucpe_cam_prep per step, through
    the C ABI with the pointers prepared once. Inputs (254 MB for the ucpe
    workload) and outputs exceed L2, so no flush is needed."""
    import ctypes as C

    import torch

    import qk_rmsnorm_rope_qknr_b200 as Q
    import workloads as W

    rank, world, local, dev, pg = init_gpu()
    L = Q.lib()
    inp = W.make_inputs(w, device=dev, seed=w.seed + rank)
    B, N, H, D = w.batch, w.seq, w.heads, w.head_dim
    act = inp["q_normed"].dtype
    outs = [torch.empty(B, H, D, N, dtype=act, device=dev) for _ in range(3)]
    infl = torch.empty(B, H, N, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    # the binding's checks once, then the bare C call for the timed steps
    Q.qknr_ucpe_cam_prep(*(inp[n] for n in UCPE_INPUTS), *outs, infl, k_scale=w.k_scale,
                         stream=stream)
    ptrs = [inp[n].data_ptr() for n in UCPE_INPUTS] + [o.data_ptr() for o in outs] + \
        [infl.data_ptr()]
    cargs = ptrs + [Q.QKNR_DT_F16 if w.act == "f16" else Q.QKNR_DT_BF16, B, N, H, D,
                    C.c_float(w.k_scale), stream.cuda_stream]

    def step(i):
        rc = L.qknr_ucpe_cam_prep(*cargs)
        if rc:
            Q._check(rc)

    ms_per_step, clocks, spread = time_steps(step, args, stream, local, dev, pg)
    tokens_per_s = world * B * N / (ms_per_step / 1e3)
    alg_bytes = W.algorithmic_bytes(w)
    peak, peak_kind = measured_peaks()
    achieved = alg_bytes / (ms_per_step / 1e3) / 1e9
    tr = TRAFFIC.get(w.name)
    traffic = tr[0] if tr and tr[1] == kernel_source_hash("ucpe") else None

    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e_ucpe(args, w, inp, outs, infl, stream, dev, world, pg)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        inp_cpu = {k: v.cpu() for k, v in inp.items()}
        n, sec, threads = oracle_sample(w, inp_cpu, args.cpu_seconds, chunk=64)
        cpu = {"value": n / sec, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": f"{n} tokens (all {H} heads each) of {w.name} in order, cycling "
                         f"through its {B * N} ({sec:.1f} s of fp64 oracle work)",
               "value_1core": one_core(w, inp_cpu, args.cpu_seconds / 4, 16)}
    if rank == 0:
        clk = clocks.summary()
        in_mb = sum(inp[n].numel() * inp[n].element_size() for n in UCPE_INPUTS) / 1e6
        line = {
            "metric": METRIC, "value": tokens_per_s, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic",
            "config": {"workload": w.name, "tokens_per_gpu": B * N, "io": f"{w.act} in and out, "
                       "f32 matrices, tables and inflation_sq",
                       "shape_in": [B, N, H, D], "shape_out": [B, H, D, N],
                       "k_scale": w.k_scale,
                       "parallelism": f"dp{world}" if world > 1 else "single",
                       "l2": f"no flush: inputs {in_mb:.0f} MB > 126 MB L2",
                       "spin_up_ms": args.spin_ms},
            "hbm_gbs": achieved, "hbm_pct_of_peak": 100.0 * achieved / peak,
            "kernel_us": ms_per_step * 1e3,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "peak_source": f"{peak_kind} hbm_gbs",
                         "algorithmic_bytes_per_launch": alg_bytes},
            "cpu_baseline": cpu, "clocks": clk, "e2e": e2e,
            "gpu_launches": args.steps, "clock_normalised": clock_normalised(ms_per_step * 1e3, clk),
            "launch_spread": spread,
        }
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    return 0


def measure_e2e_ucpe(args, w, inp, outs, infl, stream, dev, world, pg):
    """End to end through the C ABI for the camera prep, inputs and outputs in
    page-locked host memory. Three ways, the fastest reported beside the
    copies alone:
      staged:    copy the seven inputs in, run, copy the four outputs back;
      zero-copy: the kernel reads and writes the host buffers across the bus;
      pipelined: two device buffer sets and two copy streams, so that step
                 i's outputs go back while step i+1's inputs come in (a
                 token chunk's outputs would be strided in [B, H, D, N], so
                 the overlap is across steps, not inside one).
    Every step moves all of its inputs in and all of its outputs back."""
    import torch

    import qk_rmsnorm_rope_qknr_b200 as Q

    host = {n: torch.empty(inp[n].shape, dtype=inp[n].dtype).pin_memory() for n in UCPE_INPUTS}
    for n in UCPE_INPUTS:
        host[n].copy_(inp[n].cpu())
    h_out = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs + [infl]]
    d_in = {n: torch.empty_like(inp[n]) for n in UCPE_INPUTS}
    steps = max(3, min(args.e2e_steps, args.steps))

    def staged():
        for n in UCPE_INPUTS:
            d_in[n].copy_(host[n], non_blocking=True)
        Q.qknr_ucpe_cam_prep(*(d_in[n] for n in UCPE_INPUTS), *outs, infl, k_scale=w.k_scale,
                             stream=stream)
        for h, o in zip(h_out, outs + [infl]):
            h.copy_(o, non_blocking=True)

    def zero_copy():
        Q.qknr_ucpe_cam_prep(*(host[n] for n in UCPE_INPUTS), *h_out, k_scale=w.k_scale,
                             stream=stream)

    # pipelined: set k of two device buffer sets serves steps k, k+2, ...
    sets = [(d_in, outs + [infl])]
    sets.append(({n: torch.empty_like(inp[n]) for n in UCPE_INPUTS},
                 [torch.empty_like(o) for o in outs + [infl]]))
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_k = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for e in ev_out:
        e.record(s_out)
    step_no = [0]

    def pipelined():
        k = step_no[0] % 2
        step_no[0] += 1
        din, dout = sets[k]
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_k[k])      # the kernel two steps back has read these inputs
            for n in UCPE_INPUTS:
                din[n].copy_(host[n], non_blocking=True)
            ev_in[k].record(s_in)
        stream.wait_event(ev_in[k])
        stream.wait_event(ev_out[k])      # its outputs of two steps back have left
        Q.qknr_ucpe_cam_prep(*(din[n] for n in UCPE_INPUTS), *dout, k_scale=w.k_scale,
                             stream=stream)
        ev_k[k].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_k[k])
            for h, o in zip(h_out, dout):
                h.copy_(o, non_blocking=True)
            ev_out[k].record(s_out)

    def timed(step):
        for _ in range(2):
            step()
        torch.cuda.synchronize()
        if pg:
            pg.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            step()
        b.record(stream)
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / steps
        if pg:
            t = torch.tensor([ms], device=dev)
            pg.all_reduce(t, op=pg.ReduceOp.MAX)
            ms = t.item()
        return ms

    s_copy = torch.cuda.Stream(dev)

    def copies_only():
        for n in UCPE_INPUTS:
            d_in[n].copy_(host[n], non_blocking=True)
        with torch.cuda.stream(s_copy):
            for h, o in zip(h_out, outs + [infl]):
                h.copy_(o, non_blocking=True)
        stream.wait_stream(s_copy)

    def timed_pipelined():
        # as timed(), but the region ends only when the last outputs are home
        for _ in range(2):
            pipelined()
        torch.cuda.synchronize()
        if pg:
            pg.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            pipelined()
        stream.wait_stream(s_out)
        b.record(stream)
        torch.cuda.synchronize()
        ms_ = a.elapsed_time(b) / steps
        if pg:
            t = torch.tensor([ms_], device=dev)
            pg.all_reduce(t, op=pg.ReduceOp.MAX)
            ms_ = t.item()
        return ms_

    ms = {"staged": timed(staged), "zero-copy": timed(zero_copy),
          "pipelined": timed_pipelined()}
    best = min(ms, key=ms.get)
    bus_ms = timed(copies_only)
    return {"value": world * w.tokens / (ms[best] / 1e3), "unit": "tokens/s",
            "h2d_bytes_per_step": sum(inp[n].numel() * inp[n].element_size() for n in UCPE_INPUTS),
            "d2h_bytes_per_step": sum(o.numel() * o.element_size() for o in outs + [infl]),
            "steps": steps, "mode": best,
            "ms_per_step": {k: round(v, 4) for k, v in ms.items()},
            "copies_only_ms_per_step": round(bus_ms, 4),
            "frac_of_copies_only": round(bus_ms / ms[best], 4)}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="qknr", choices=["qknr", "reference"])
    ap.add_argument("--workload", default="fp8neox")
    ap.add_argument("--spin-ms", type=float, default=1000.0,
                    help="untimed steps for this long before the warm-up, with the clock "
                         "sampler running")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--host-sweep", action="store_true",
                    help="print host cost against device time per call, 64-8192 tokens")
    ap.add_argument("--tokens", type=int, default=None,
                    help="run the workload's geometry on this many tokens instead (3D: a "
                         "sequence shard from position 0); for profiling smaller cases")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    import workloads as W

    w = W.WORKLOADS[args.workload]
    if args.tokens:
        import dataclasses

        if w.form == "3d":
            w = dataclasses.replace(w, name=f"{w.name}[{args.tokens}]", batch=1, seq=args.tokens,
                                    input_2d=True)
        elif w.form == "ucpe":
            w = dataclasses.replace(w, name=f"{w.name}[{args.tokens}]", seq=args.tokens)
        else:
            w = dataclasses.replace(w, name=f"{w.name}[{args.tokens}]", tokens=args.tokens)
    if args.impl == "reference":
        return run_reference(args, w)
    if args.host_sweep:
        return run_host_sweep(args)
    if w.form == "ucpe":
        return run_gpu_ucpe(args, w)
    return run_gpu(args, w) if w.form == "3d" else run_gpu_table(args, w)


if __name__ == "__main__":
    sys.exit(main())
