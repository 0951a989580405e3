"""Benchmark of the EFLA forward hot path on B200.

One step = one pass of the whole hot path over one batch of the 1.3B-LM-shaped
workload: the chunkwise forward (B=4, H=16, L=4096, dk=dv=128, chunk=64, bf16,
o written at the input dtype unless --o-dtype fp32) followed by the recurrent
decode step of its decode batch (B=64, H=16, one token each, fp32 carried
state).  Throughput is token-heads per second
(B*H*L + B_dec*H_dec per step).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload 3|4|5] [--no-e2e] [--no-cpu-baseline]
                    [--o-dtype input|fp32] [--gated] [--rule exact|euler] [--pass fwd|bwd]

Under torchrun (WORLD_SIZE > 1) every rank runs its own replica of the workload
on disjoint heads (seeded per rank): heads are independent, so there is no
collective on the data path ("weak" scaling); the only collectives are the
barriers around the timed region and the max-reduction of its time.

Prints ONE JSON line (rank 0).
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

import torch  # noqa: E402

from delta_rule_linear_efla_b200 import dist as edist  # noqa: E402
from delta_rule_linear_efla_b200 import inputs  # noqa: E402

METRIC = "EFLA fwd tokens/s per GPU (B*H*L/time) and % of binding roofline"
UNIT = "token-heads/s"


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sus=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


def alg_bytes_chunk(w, o_bytes: int | None = None) -> int:
    """Algorithmic HBM bytes of one chunk forward: read q, k, v, beta and write o per
    token-head, plus the fp32 final state per head (S0 is zero here and not read).  By default
    o is counted at the input dtype, the count of the hot-path scope table (1026 B per
    token-head at dk = dv = 128 in bf16); o_bytes = 4 counts the fp32 output the library
    writes by default."""
    es = 2 if w.dtype == "bf16" else 4
    ob = es if o_bytes is None else o_bytes
    per_tok = (2 * w.dk + w.dv) * es + es + w.dv * ob + (es if GATED else 0)  # + the decay g
    return w.token_heads * per_tok + w.B * w.H * w.dk * w.dv * 4


def alg_bytes_bwd(w) -> int:
    """Algorithmic HBM bytes of one backward call: read q, k, v, beta (input dtype) and dO
    (fp32), write dq, dk, dv (fp32) and dbeta (fp32) per token-head; S0 is zero here and
    dS_final is not given."""
    es = 2 if w.dtype == "bf16" else 4
    per_tok = (2 * w.dk + w.dv) * es + es + w.dv * 4 + (2 * w.dk + w.dv) * 4 + 4
    return w.token_heads * per_tok


def run_bwd(args) -> None:
    """--pass bwd: the backward pass (efla_bwd) timed on the workload, one GPU."""
    from delta_rule_linear_efla_b200 import efla

    dev = torch.device("cuda", 0)
    w = inputs.WORKLOADS[args.workload]
    x = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inputs.make_inputs(w).items()}
    g = torch.Generator().manual_seed(77)
    dO = torch.randn(w.B, w.H, w.L, w.dv, generator=g).to(dev)
    ws = torch.empty(max(1, efla.load_library().efla_bwd_workspace_size(w.B, w.H, w.L, w.dk, w.dv)),
                     dtype=torch.uint8, device=dev)
    call = lambda: efla.bwd(x["q"], x["k"], x["v"], x["beta"], dO, x["S0"], None, want_dS0=False,
                            rule=RULE, workspace=ws)
    for _ in range(max(3, args.warmup)):
        call()
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = ClockSampler(0)
    clk.start()
    l0 = efla.kernel_launches()
    a.record()
    for _ in range(args.steps):
        call()
    b.record()
    torch.cuda.synchronize(dev)
    launches = efla.kernel_launches() - l0
    clocks = clk.stop()
    ms = a.elapsed_time(b) / args.steps
    # a training step, forward then backward: chunk_fwd + bwd against the pair that keeps the
    # forward's values for the backward (chunk_fwd_keep + bwd(kept=...)), o at the input dtype
    train = None
    if efla.keeps_for_bwd(x["q"], x["v"], rule=RULE):
        o_dt = _o_dtype(w)

        def plain_step():
            efla.chunk_fwd(x["q"], x["k"], x["v"], x["beta"], x["S0"], o_dtype=o_dt, rule=RULE)
            call()

        def keep_step():
            _, _, kept = efla.chunk_fwd_keep(x["q"], x["k"], x["v"], x["beta"], x["S0"], o_dtype=o_dt, rule=RULE)
            efla.bwd(x["q"], x["k"], x["v"], x["beta"], dO, x["S0"], None, want_dS0=False, rule=RULE,
                     workspace=ws, kept=kept)

        train = {}
        for name, f in (("ms_fwd_then_bwd", plain_step), ("ms_fwd_keep_then_bwd_kept", keep_step)):
            for _ in range(3):
                f()
            torch.cuda.synchronize(dev)
            a.record()
            for _ in range(args.steps):
                f()
            b.record()
            torch.cuda.synchronize(dev)
            train[name] = a.elapsed_time(b) / args.steps
        train["token_heads_per_s"] = w.token_heads / (train["ms_fwd_keep_then_bwd_kept"] / 1e3)
    alg = alg_bytes_bwd(w)
    peaks = _peaks()
    achieved = alg / (ms / 1e3) / 1e9
    print(json.dumps({
        "metric": "EFLA bwd tokens/s per GPU (B*H*L/time) and % of binding roofline", "value":
        w.token_heads / (ms / 1e3), "unit": UNIT, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic", "config": _config(w),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm"],
                     "traffic": profiled_bwd_traffic(w) if RULE == "exact" else None,
                     "kernel": "efla_bwd (bf16 heads the saved-forward gate admits: the saving tensor-core "
                               "forward, the reverse chain over chunks on tcgen05, per-chunk gradients on "
                               "tcgen05 at d = 128 and mma.sync at d = 64; other heads: the fp32 "
                               "column-block walk on CUDA cores)",
                     "alg_bytes_per_launch": alg, "avg_launch_ms": ms,
                     "source_hash": kernel_source_hash(BWD_SOURCES)},
        "train_step": train, "gpu_launches": int(launches), "clocks": clocks}))


def alg_bytes_decode(Bd, Hd, dk, dv, es=2) -> int:
    """Read + write of the fp32 state per head, plus q, k, v, beta in and o out."""
    return Bd * Hd * (2 * dk * dv * 4 + (2 * dk + 2 * dv + 1) * es)


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            import tempfile

            fd, self.path = tempfile.mkstemp(prefix="efla_bench_clocks_", suffix=".csv")
            self.f = os.fdopen(fd, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            lines = f.readlines()
        os.remove(self.path)
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


FWD_SOURCES = ("chunk_tc.cu", "common.cuh", "tc_ptx.cuh", "tmap.h")
# the backward's kernels: its own sources and the saving forward's
BWD_SOURCES = FWD_SOURCES + ("backward.cu", "bwd_tc.cu", "bwd_gate.cuh")


def kernel_source_hash(files=FWD_SOURCES) -> str:
    """Hash of the CUDA sources a pass's kernels are built from (for the chunk forward: the
    tcgen05 pair and segment kernels and the helpers they include): ties profiled counters to
    them."""
    import hashlib

    h = hashlib.sha256()
    for f in files:
        h.update(f.encode())
        h.update(open(os.path.join(ROOT, "delta_rule_linear_efla_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def _profile_keys(name: str) -> dict:
    p = os.path.join(ROOT, "profiles", name)
    kv = {}
    if os.path.exists(p):
        for line in open(p):
            line = line.split("#")[0].strip()
            if "=" in line:
                k, v = (x.strip() for x in line.split("=", 1))
                kv[k] = v
    return kv


def profiled_bwd_traffic(w) -> int | None:
    """DRAM bytes of one efla_bwd call from the committed ncu capture, if it was taken on this
    workload and on the current backward sources; None otherwise."""
    if w.id != 4:
        return None
    kv = _profile_keys("dram_traffic_bwd_lm1p3b.txt")
    if kv.get("source_hash") != kernel_source_hash(BWD_SOURCES) or "bwd_bytes" not in kv:
        return None
    return int(kv["bwd_bytes"])


def profiled_traffic(w, o_dtype) -> int | None:
    """DRAM bytes of one efla_chunk_fwd call from the committed ncu capture, if it was taken on
    this workload, with this output dtype and on the current kernel sources; None otherwise."""
    if w.id != 4:
        return None
    p = os.path.join(ROOT, "profiles", "dram_traffic_lm1p3b.txt")
    if not os.path.exists(p):
        return None
    kv = {}
    for line in open(p):
        line = line.split("#")[0].strip()
        if "=" in line:
            k, v = (x.strip() for x in line.split("=", 1))
            kv[k] = v
    if kv.get("source_hash") != kernel_source_hash() or kv.get("o_dtype", "fp32") != _o_name(o_dtype):
        return None
    return int(kv["chunk_fwd_bytes"])


def cpu_baseline(w, seconds_target: float = 12.0) -> dict:
    """The fp64 oracle (as it stands) on a bounded sample of the workload: a subset of its
    heads at full sequence length, on all host cores."""
    import oracle

    oracle.build()
    cores = os.cpu_count() or 1
    x = _with_gate(inputs.make_inputs(inputs.workload(w.id, B=1, H=1)), 7)
    t0 = time.perf_counter()
    oracle.fwd(x["q"], x["k"], x["v"], x["beta"], x["S0"], nthreads=1, rule=RULE, g=x.get("g"))
    t_head = max(time.perf_counter() - t0, 1e-3)
    # about `seconds_target` of wall time with every core busy on whole heads
    heads = max(1, min(w.B * w.H, cores * max(1, int(seconds_target / t_head))))
    H = min(heads, w.H)
    B = max(1, min(w.B, heads // H))
    xs = _with_gate(inputs.make_inputs(inputs.workload(w.id, B=B, H=H)), 8)
    threads = min(cores, B * H)
    # repeat the sample until it amounts to ~seconds_target of CPU work (core-seconds)
    reps, dt = 0, 0.0
    t0 = time.perf_counter()
    while reps < 50 and (reps == 0 or dt * threads < seconds_target):
        oracle.fwd(xs["q"], xs["k"], xs["v"], xs["beta"], xs["S0"], nthreads=threads, rule=RULE,
                   g=xs.get("g"))
        reps += 1
        dt = time.perf_counter() - t0
    n = B * H * w.L * reps
    return {"value": n / dt, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": "%d of %d heads (B=%d, H=%d) at full L=%d, %d pass(es), fp64 token-by-token, "
                      "%.1f s on %d threads" % (B * H, w.B * w.H, B, H, w.L, reps, dt, threads)}


def run_reference(args) -> None:
    """The oracle timed on host cores: each step is a bounded sample of the workload."""
    ws, rank, _ = edist.world()
    if rank != 0:
        return
    import oracle

    oracle.build()
    w = inputs.WORKLOADS[args.workload]
    cores = os.cpu_count() or 1
    bwd = args.pass_ == "bwd"
    # the backward oracle runs heads one after another (it keeps every state): a smaller sample
    H = min(w.H, 2 if bwd else cores)
    xs = _with_gate(inputs.make_inputs(inputs.workload(w.id, B=1, H=H, L=min(w.L, 512 if bwd else 1024))), 9)
    threads = 1 if bwd else min(cores, H)
    if bwd:
        dO = torch.randn(xs["v"].shape, generator=torch.Generator().manual_seed(77), dtype=torch.float64)
        run = lambda: oracle.bwd(xs["q"], xs["k"], xs["v"], xs["beta"], dO, xs["S0"], None, rule=RULE)
    else:
        run = lambda: oracle.fwd(xs["q"], xs["k"], xs["v"], xs["beta"], xs["S0"], nthreads=threads,
                                 rule=RULE, g=xs.get("g"))
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    dt = time.perf_counter() - t0
    n = H * xs["q"].shape[2] * args.steps
    val = n / dt
    sample = "%d heads x L=%d of workload %s per step, fp64 token-by-token%s" % (
        H, xs["q"].shape[2], w.name, " (backward)" if bwd else "")
    metric = "EFLA bwd tokens/s per GPU (B*H*L/time) and % of binding roofline" if bwd else METRIC
    print(json.dumps({
        "impl": "reference", "metric": metric, "value": val, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": _config(w),
        "cpu_baseline": {"value": val, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


RULE = "exact"  # set from --rule: "exact" (the method) or "euler" (the delta rule, for comparison)
GATED = False  # set from --gated: the gated form, a per-token decay g_t ~ sigmoid(N(2, 1))
O_DT = "input"  # set from --o-dtype: o at the input dtype (default) or fp32


def _with_gate(x: dict, seed: int) -> dict:
    """The inputs with the gated form's per-token decay added (when --gated)."""
    if GATED:
        x["g"] = inputs.make_gate(x["beta"].shape, x["beta"].dtype, seed)
    return x


def _o_dtype(w):
    """The output dtype of the timed calls: the input dtype by default (o at the input dtype, as
    the algorithmic byte count has it), fp32 with --o-dtype fp32."""
    return torch.float32 if (O_DT == "fp32" or w.dtype != "bf16") else torch.bfloat16


def _o_name(dt) -> str:
    return "fp32" if dt == torch.float32 else "bf16"


def _config(w) -> dict:
    c = {"workload": "%s (B=%d H=%d L=%d dk=%d dv=%d chunk=%d %s)" % (
        w.name, w.B, w.H, w.L, w.dk, w.dv, w.chunk, w.dtype),
        "B": w.B, "H": w.H, "L": w.L, "dk": w.dk, "dv": w.dv, "chunk": w.chunk,
        "l2": "inputs > L2 (126 MB): two rotating input sets per rank",
        "o_dtype": _o_name(_o_dtype(w)), "rule": RULE}
    if GATED:
        c["gate"] = "g_t ~ sigmoid(N(2, 1)) per token: S_t = g_t (I - a k k^T) S + a k v^T"
    if w.decode:
        c["decode"] = "B=%d H=%d one token, fp32 carried state" % (w.decode["B"], w.decode["H"])
    return c


def _roofline(w, chunk_ms: float, peaks: dict, path: str, o_dtype=torch.float32) -> dict:
    """HBM roofline of one efla_chunk_fwd call from its CUDA-event time.  `frac` counts the
    algorithmic bytes with o at the input dtype (the hot-path scope table's count); the
    `fp32_output` entry counts o at 4 bytes, what the call writes with an fp32 output."""
    alg = alg_bytes_chunk(w)
    achieved = alg / (chunk_ms / 1e3) / 1e9
    r = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm"], "unit": "GB/s",
         "frac": achieved / peaks["hbm"], "alg_bytes_per_launch": alg, "avg_launch_ms": chunk_ms,
         "kernel": "efla_chunk_fwd (%s path), o written as %s" % (
             path, "fp32" if o_dtype == torch.float32 else "bf16"),
         "peak_source": peaks["src"] + " (MEASURED_PEAKS.json hbm_gbs, copy burst)"}
    if o_dtype == torch.float32:
        alg32 = alg_bytes_chunk(w, o_bytes=4)
        a32 = alg32 / (chunk_ms / 1e3) / 1e9
        r["fp32_output"] = {"alg_bytes_per_launch": alg32, "achieved": a32, "frac": a32 / peaks["hbm"]}
    return r


def time_chunk_fwd(w, dev, peaks: dict, steps: int, o_dtype=torch.float32) -> dict:
    """efla_chunk_fwd alone on a workload: two rotating input sets (larger than L2 together),
    3 warm-up calls, then `steps` calls each timed with CUDA events on the launching stream."""
    from delta_rule_linear_efla_b200 import efla

    sets = []
    for r in range(2):
        x = _with_gate(inputs.make_inputs(w, seed=1000 + w.id + 17 * r), 500 + r)
        sets.append({k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()})
    o_buf = [torch.empty((w.B, w.H, w.L, w.dv), dtype=o_dtype, device=dev) for _ in range(2)]
    Sf = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device=dev)
    wsb = efla.workspace_size(w.B, w.H, w.L, w.dk, w.dv, w.chunk, w.torch_dtype(), o_dtype)
    wsp = torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev)
    path = efla.chunk_fwd_path(w.B, w.H, w.L, w.dk, w.dv, w.chunk, w.torch_dtype(), o_dtype)
    stream = torch.cuda.current_stream(dev)

    def call(i):
        x = sets[i % 2]
        efla.chunk_fwd(x["q"], x["k"], x["v"], x["beta"], x["S0"], chunk=w.chunk, o=o_buf[i % 2],
                       S_final=Sf, workspace=wsp, o_dtype=o_dtype, rule=RULE, g=x.get("g"))

    for i in range(3):
        call(i)
    torch.cuda.synchronize(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for i, (a, b) in enumerate(evs):
        a.record(stream)
        call(i)
        b.record(stream)
    torch.cuda.synchronize(dev)
    if efla.last_device_error() != 0:
        raise RuntimeError("device error word set")
    ms = [a.elapsed_time(b) for a, b in evs]
    mean = sum(ms) / len(ms)
    r = _roofline(w, mean, peaks, path, o_dtype)
    r.update({"workload": _config(w)["workload"], "ms": mean, "ms_min": min(ms),
              "token_heads_per_s": w.token_heads / (mean / 1e3), "steps": steps})
    del sets, o_buf, wsp
    torch.cuda.empty_cache()
    return r


def run_ours(args) -> None:
    from delta_rule_linear_efla_b200 import efla

    ws, rank, local = edist.world()
    if ws > 1:
        torch.cuda.set_device(local)
        edist.init("nccl", timeout_s=120)
    dev = torch.device("cuda", local if ws > 1 else 0)
    torch.cuda.set_device(dev)
    w = inputs.WORKLOADS[args.workload]
    peaks = _peaks()

    # ---- inputs: two rotating sets so consecutive steps do not hit in L2 ----
    sets = []
    for r in range(2):
        x = _with_gate(inputs.make_inputs(w, seed=edist.replica_seed(1000 + w.id, rank, r)),
                       edist.replica_seed(600, rank, r))
        sets.append({k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()})
    odt = _o_dtype(w)
    o_buf = [torch.empty((w.B, w.H, w.L, w.dv), dtype=odt, device=dev) for _ in range(2)]
    Sf_buf = [torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device=dev) for _ in range(2)]
    ws_bytes = efla.workspace_size(w.B, w.H, w.L, w.dk, w.dv, w.chunk, w.torch_dtype(), odt)
    wsp = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    path = efla.chunk_fwd_path(w.B, w.H, w.L, w.dk, w.dv, w.chunk, w.torch_dtype(), odt)

    dec = None
    if w.decode:
        d = inputs.make_decode_inputs(w, seed=edist.replica_seed(w.decode["seed"], rank))
        dd = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()
              if k != "prefix"}
        p = d["prefix"]
        pd = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in p.items()}
        _, S_carry = efla.chunk_fwd(pd["q"], pd["k"], pd["v"], pd["beta"], None, chunk=w.chunk,
                                    rule=RULE)
        if GATED:
            dd["g"] = inputs.make_gate((w.decode["B"], w.decode["H"]), w.torch_dtype(), 700 + rank).to(dev)
        dd["S_init"] = S_carry
        dd["S"] = [S_carry.clone(), S_carry.clone()]
        dd["o"] = torch.empty((w.decode["B"], w.decode["H"], w.dv), dtype=odt, device=dev)
        dec = dd
    tok_dec = (w.decode["B"] * w.decode["H"]) if w.decode else 0
    tok_step = w.token_heads + tok_dec

    stream = torch.cuda.current_stream(dev)

    def step(i, ev_pair=None):
        x = sets[i % 2]
        if ev_pair is not None:
            ev_pair[0].record(stream)
        efla.chunk_fwd(x["q"], x["k"], x["v"], x["beta"], x["S0"], chunk=w.chunk,
                       o=o_buf[i % 2], S_final=Sf_buf[i % 2], workspace=wsp, rule=RULE, g=x.get("g"))
        if ev_pair is not None:
            ev_pair[1].record(stream)
        if dec is not None:
            efla.recurrent_step(dec["q"], dec["k"], dec["v"], dec["beta"], dec["S"][i % 2],
                                o=dec["o"], rule=RULE, g=dec.get("g"))

    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize(dev)
    edist.barrier()
    torch.cuda.synchronize(dev)

    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = ClockSampler(dev.index if dev.index is not None else 0)
    clk.start()
    l0 = efla.kernel_launches()
    t_start.record(stream)
    for i in range(args.steps):
        step(i, evs[i])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    launches = efla.kernel_launches() - l0
    clocks = clk.stop()
    edist.barrier()
    ms_local = t_start.elapsed_time(t_end)
    ms = edist.max_over_ranks(ms_local, dev)
    chunk_ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
    chunk_ms = edist.max_over_ranks(chunk_ms, dev)
    err = efla.last_device_error()
    if err != 0:
        raise RuntimeError("device error word set: %s" % efla.status_str(err))

    value = edist.aggregate_rate(tok_step, args.steps, ws, ms)
    roofline = _roofline(w, chunk_ms, peaks, path, odt)
    roofline["traffic"] = profiled_traffic(w, odt)
    roofline["source_hash"] = kernel_source_hash()

    # ---- end to end through the public API with host buffers ----
    e2e = None
    if not args.no_e2e:
        xh = {k: (v.pin_memory() if isinstance(v, torch.Tensor) else v)
              for k, v in _with_gate(inputs.make_inputs(w, seed=4242 + rank), 4343 + rank).items()}
        o_host = torch.empty((w.B, w.H, w.L, w.dv), dtype=odt).pin_memory()
        S_host = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32).pin_memory()
        names = ("q", "k", "v", "beta") + (("g",) if GATED else ())
        h2d = sum(xh[k].numel() * xh[k].element_size() for k in names)
        d2h = o_host.numel() * o_host.element_size() + S_host.numel() * 4
        if dec is not None:
            dh = {k: dec[k].cpu().pin_memory() for k in ("q", "k", "v", "beta") + (("g",) if GATED else ())}
            S_dec_host = dec["S_init"].cpu().pin_memory()
            od_host = torch.empty_like(dec["o"], device="cpu").pin_memory()
            h2d += sum(t.numel() * t.element_size() for t in dh.values()) + S_dec_host.numel() * 4
            d2h += od_host.numel() * od_host.element_size() + S_dec_host.numel() * 4

        # Steps are pipelined the way a user of the API would: two device buffer sets, uploads on
        # one copy stream and downloads on another, so step i+1's upload and step i's download
        # overlap step i's kernels.  Every step still moves its own inputs in and results out.
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        din = [{k: torch.empty_like(xh[k], device=dev) for k in names} for _ in range(2)]
        o_host2 = [o_host, torch.empty_like(o_host).pin_memory()]
        S_host2 = [S_host, torch.empty_like(S_host).pin_memory()]
        if dec is not None:
            ddin = [{k: torch.empty_like(dh[k], device=dev) for k in dh} for _ in range(2)]
            Sd2 = [torch.empty_like(S_dec_host, device=dev) for _ in range(2)]
            od2 = [torch.empty_like(dec["o"]) for _ in range(2)]
            od_host2 = [od_host, torch.empty_like(od_host).pin_memory()]
            Sdo_host2 = [torch.empty_like(S_dec_host).pin_memory() for _ in range(2)]
        ev = {n: [torch.cuda.Event() for _ in range(2)] for n in ("in_ready", "in_free", "done", "out_free")}

        def e2e_step(i):
            j = i % 2
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev["in_free"][j])  # step i-2's kernels are done with din[j]
                for k in names:
                    din[j][k].copy_(xh[k], non_blocking=True)
                if dec is not None:
                    for k in dh:
                        ddin[j][k].copy_(dh[k], non_blocking=True)
                    Sd2[j].copy_(S_dec_host, non_blocking=True)
                ev["in_ready"][j].record(s_in)
            stream.wait_event(ev["in_ready"][j])
            stream.wait_event(ev["out_free"][j])  # step i-2's downloads are done with the outputs
            g = din[j]
            efla.chunk_fwd(g["q"], g["k"], g["v"], g["beta"], None, chunk=w.chunk, o=o_buf[j],
                           S_final=Sf_buf[j], workspace=wsp, rule=RULE, g=g.get("g"))
            if dec is not None:
                gd = ddin[j]
                efla.recurrent_step(gd["q"], gd["k"], gd["v"], gd["beta"], Sd2[j], o=od2[j], rule=RULE,
                                    g=gd.get("g"))
            ev["in_free"][j].record(stream)
            ev["done"][j].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev["done"][j])
                o_host2[j].copy_(o_buf[j], non_blocking=True)
                S_host2[j].copy_(Sf_buf[j], non_blocking=True)
                if dec is not None:
                    od_host2[j].copy_(od2[j], non_blocking=True)
                    Sdo_host2[j].copy_(Sd2[j], non_blocking=True)
                ev["out_free"][j].record(s_out)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        edist.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(3, min(args.steps, 10))
        a.record(stream)
        for i in range(n_e2e):
            e2e_step(i)
        stream.wait_stream(s_out)  # the last step's downloads are inside the timed region
        b.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = edist.max_over_ranks(a.elapsed_time(b), dev)
        e2e = {"value": edist.aggregate_rate(tok_step, n_e2e, ws, e_ms), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "steps": n_e2e, "ms_per_step": e_ms / n_e2e}

    per_workload = None
    if ws == 1 and not args.no_per_workload:
        per_workload = {}
        for wid in (3, 4, 5):
            if wid != w.id:
                ow = inputs.WORKLOADS[wid]
                per_workload[str(wid)] = time_chunk_fwd(ow, dev, peaks, args.steps, o_dtype=_o_dtype(ow))
        # the headline workload with the other output dtype
        other = torch.float32 if odt == torch.bfloat16 else torch.bfloat16
        if w.dtype == "bf16":
            per_workload["%d_o_%s" % (w.id, _o_name(other))] = time_chunk_fwd(
                w, dev, peaks, args.steps, o_dtype=other)

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w)

    if ws > 1:
        import torch.distributed as dist

        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic", "config": _config(w), "roofline": roofline, "cpu_baseline": cpu,
        "e2e": e2e, "gpu_launches": int(launches), "clocks": clocks,
        "path": path, "token_heads_per_step": tok_step, "per_workload": per_workload,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, default=4, choices=[2, 3, 4, 5])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--gated", action="store_true",
                    help="the gated form: a per-token decay g_t ~ sigmoid(N(2, 1)) on the carried state")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="skip timing the other workloads' chunk forward after the timed region")
    ap.add_argument("--o-dtype", choices=["input", "fp32"], default="input",
                    help="output dtype of the timed chunk forward and decode: the input dtype "
                         "(default; the algorithmic byte count's o) or fp32")
    ap.add_argument("--pass", dest="pass_", choices=["fwd", "bwd"], default="fwd",
                    help="fwd (default): the forward step; bwd: the backward pass alone")
    ap.add_argument("--rule", choices=["exact", "euler"], default="exact",
                    help="update rule: the exact flow (default) or the delta rule's Euler step, "
                         "for the throughput comparison (the workload's keys are not normalised, "
                         "so under euler only the time is meaningful)")
    args = ap.parse_args()
    global RULE, GATED, O_DT
    RULE = args.rule
    GATED = args.gated
    O_DT = args.o_dtype
    if args.warmup < 3:
        args.warmup = 3
    if args.gated and args.pass_ == "bwd":
        raise SystemExit("--pass bwd: the backward pass is for the ungated form")
    if args.impl == "reference":
        run_reference(args)
    elif args.pass_ == "bwd":
        run_bwd(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
