"""Benchmark of the B200 BitLinear (W1.58A8) path.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference]

One step is one pass of the hot path over one batch of synthetic input: the
prefill workload of the 2B model's projection shapes, M = 4096 tokens through
(K, N) = (2560, 6912) and (6912, 2560), each as RMSNorm prelude + per-token
int8 quant (bitnet_quant_act) followed by the int8 x ternary contraction with
its bf16 dequant epilogue (bitnet_linear).  The packed weights are prepared
once (the pages' packed checkpoint stores them ternary, "offline").

Prints ONE JSON line (rank 0).  `value` is int8 TOPS (2*M*N*K per projection,
zero weights not skipped) over all ranks; `roofline` is the tcgen05 GEMM's
achieved fraction of the int8 tensor peak; `e2e` is the same step through the
C ABI with host buffers (pinned H2D of the activations, D2H of the outputs,
pipelined over token chunks on two copy streams);
`cpu_baseline` is the CPU oracle on a bounded sample of the same step;
`workloads` adds the decode GEMV streaming bandwidth and the FFN / H-FFN /
tiny configurations.

Under torchrun (N > 1) every rank runs the same step on its own GPU (the
projection is independent per token, so tokens shard with no data-path
collective: weak scaling); the elapsed time is the max over ranks.
`--impl reference` times the CPU oracle instead (rank 0 only).
"""
import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic  # noqa: E402

METRIC = "BitLinear W1.58A8 int8 TOPS (prefill) & GB/s (decode), % of roofline on 1 B200"
PREFILL_M = 4096
PREFILL_KN = ((2560, 6912), (6912, 2560))
DECODE_M = (1, 4, 16)
DECODE_KN = ((2560, 2560), (2560, 6912), (6912, 2560))
# the prefill GEMM kernel and the headers whose device code it compiles in
GEMM_KERNEL_SRCS = [os.path.join(ROOT, "ternary_weight_token_b200", "csrc", n)
                    for n in ("gemm_tc.cuh", "gemv.cuh", "common.cuh")]
GEMM_PROFILE = os.path.join(ROOT, "profiles", "gemm_tc_prefill_4096x2560x6912.md")


def prefill_ops():
    return sum(2 * PREFILL_M * N * K for K, N in PREFILL_KN)


# token chunks of the end-to-end step's copy / compute / copy pipeline
E2E_CHUNKS = 8


def decode_bytes(M, K, N):
    """Algorithmic bytes of one decode call: packed weights + codes + scales +
    bf16 outputs + gamma."""
    return N * K // 4 + M * K + 4 * M + 2 * M * N + 4


# ------------------------------------------------------------ distributed

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, backend):
    if world <= 1:
        return None
    import datetime

    import torch.distributed as dist
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(value, dist, device=None):
    if dist is None:
        return value
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi while running."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="bench_clocks_", suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu_index), "-lms", "50"], stdout=self.out,
                stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        self.t0 = time.time()

    def stop(self, window):
        if self.proc is None:
            return None
        time.sleep(0.06)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                    ts += float("0." + parts[0].split(".")[1]) if "." in parts[0] else 0.0
                    rows.append((ts, float(parts[2]), float(parts[3]), parts[5:]))
                except (ValueError, IndexError):
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        t_start, t_end = window
        inside = [r for r in rows if t_start - 0.05 <= r[0] <= t_end + 0.05]
        note = "samples inside the timed region"
        if not inside:
            inside = rows
            note = "timed region shorter than the 50 ms sample period: samples around it"
        names = ["active", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        reasons = set()
        for r in inside:
            for name, val in zip(names[1:], r[3][1:]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r[1] for r in inside),
                "sm_max_mhz": max(r[2] for r in inside), "reasons": sorted(reasons),
                "samples": len(inside), "note": note}


# ------------------------------------------------------------- references

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def files_sha(paths):
    """One hash over several files' names and contents."""
    h = hashlib.sha256()
    for path in paths:
        with open(path, "rb") as f:
            h.update(os.path.basename(path).encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def nvtx_push(torch, name):
    """Named range for profilers; a no-op where NVTX is unavailable."""
    try:
        torch.cuda.nvtx.range_push(name)
    except Exception:             # noqa: BLE001
        pass


def nvtx_pop(torch):
    try:
        torch.cuda.nvtx.range_pop()
    except Exception:             # noqa: BLE001
        pass


def sources_sha():
    """One hash over the kernel sources and the C header, identifying the
    build a line was measured with."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "ternary_weight_token_b200", "csrc")
    names = sorted(n for n in os.listdir(csrc) if n.endswith((".cu", ".cuh", ".h")))
    for name in names + ["../../include/bitnet.h"]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per GEMM launch from the committed ncu summary, or None when
    the summary is missing or the kernel source changed since the capture."""
    if not os.path.exists(GEMM_PROFILE):
        return None
    txt = open(GEMM_PROFILE).read()
    m_sha = re.search(r"kernel_sources_sha256_16:\s*([0-9a-f]{16})", txt)
    m_b = re.search(r"dram_bytes_per_launch:\s*([0-9]+)", txt)
    if not m_sha or not m_b or m_sha.group(1) != files_sha(GEMM_KERNEL_SRCS):
        return None
    return int(m_b.group(1))


# ---------------------------------------------------------- CPU reference

def oracle_prefill_sample(target_s=12.0, max_tokens=PREFILL_M):
    """Time the oracle on a bounded token sample of the prefill step."""
    import oracle
    threads = oracle.num_threads()
    prepared = []
    for i, (K, N) in enumerate(PREFILL_KN):
        inp = synthetic.linear_inputs(PREFILL_M, K, N, seed=i)
        g, T, _ = oracle.quantize_weights(inp["W"])
        prepared.append((K, N, inp["X"], T, g))

    def run(tokens):
        t0 = time.perf_counter()
        for K, N, X, T, g in prepared:
            y = oracle.bitlinear(X[:tokens], T, g, oracle.PRELUDE_RMSNORM, eps=1e-5)
            oracle.round_bf16(y)
        return time.perf_counter() - t0

    run(4)                                    # warm the oracle (page faults, threads)
    tokens, dt = 8, run(8)
    while dt < target_s and tokens < max_tokens:
        tokens = int(min(max_tokens, max(2 * tokens, tokens * target_s / max(dt, 1e-3) * 1.05)))
        dt = run(tokens)
    ops = sum(2 * tokens * N * K for K, N in PREFILL_KN)
    return {"value": ops / dt / 1e12, "unit": "TOPS", "cores": threads, "kind": "oracle",
            "sample": f"{tokens} of the {PREFILL_M} tokens of one prefill step (both "
                      f"projections: RMSNorm + int8 quant + int64 contraction + fp64 dequant + "
                      f"bf16 round), {dt:.1f} s on {threads} OpenMP threads"}


def _timed(fn, min_s):
    """Run fn until min_s seconds have passed (at least twice); seconds per run."""
    fn()                                         # warm (page faults, thread pool)
    n, t0 = 0, time.perf_counter()
    while True:
        fn()
        n += 1
        dt = time.perf_counter() - t0
        if dt >= min_s and n >= 2:
            return dt / n


def oracle_workload_baselines(per_case_s=0.6):
    """The CPU oracle timed on this host for every secondary workload, on the
    same synthetic inputs (seeds) as the GPU lines: the tiny linear and the
    decode calls on one thread (a token or a few), the FFN block and the
    H-FFN on all OpenMP threads over a bounded token sample, scaled to a full
    call.  Reported baselines, not targets."""
    import oracle
    out = {}
    prev = oracle.num_threads()
    try:
        oracle.set_threads(1)
        d = synthetic.WORKLOADS["tiny"].dims
        inp = synthetic.linear_inputs(d["M"], d["K"], d["N"], seed=0)
        g, T, _ = oracle.quantize_weights(inp["W"])
        dt = _timed(lambda: oracle.bitlinear(inp["X"], T, g), per_case_s)
        out["tiny"] = {"us_per_call": dt * 1e6, "cores": 1, "kind": "oracle",
                       "sample": "the whole call (quant + contraction + dequant), 1 thread"}
        dec = []
        for K, N in DECODE_KN:
            inp = synthetic.linear_inputs(max(DECODE_M), K, N, seed=K + N)
            g, T, _ = oracle.quantize_weights(inp["W"])
            for M in DECODE_M:
                q, s, _ = oracle.quant_act(inp["X"][:M])
                dt = _timed(lambda: oracle.round_bf16(oracle.dequant(oracle.contract(q, T), s, g)),
                            per_case_s / 3)
                dec.append({"M": M, "K": K, "N": N, "us_per_call": dt * 1e6,
                            "GB_s": decode_bytes(M, K, N) / dt / 1e9, "cores": 1,
                            "kind": "oracle", "sample": "the whole call (contraction + dequant "
                                                        "+ bf16 round of int8 codes), 1 thread"})
        out["decode"] = dec
        oracle.set_threads(prev)
        d = synthetic.WORKLOADS["hffn"].dims
        inp = synthetic.hffn_inputs(d["M"], d["D"], d["F"], seed=0)
        g1, T1, _ = oracle.quantize_weights(inp["W1"])
        g2, T2, _ = oracle.quantize_weights(inp["W2"])
        rows = 128
        dt = _timed(lambda: oracle.hffn(inp["X"][:rows], T1, g1, T2, g2), per_case_s)
        full = dt * d["M"] / rows
        out["hffn"] = {"us": full * 1e6, "TOPS": 2 * 2 * d["M"] * d["D"] * d["F"] / full / 1e12,
                       "cores": prev, "kind": "oracle",
                       "sample": f"{rows} of {d['M']} tokens, scaled to the full call"}
        d = synthetic.WORKLOADS["ffn"].dims
        inp = synthetic.ffn_inputs(d["M"], d["H"], d["I"], seed=0)
        Tw = {k: oracle.quantize_weights(inp[k]) for k in ("Wg", "Wu", "Wd")}
        rows = 32
        dt = _timed(lambda: oracle.round_bf16(oracle.ffn_relu2(
            inp["x"][:rows], Tw["Wg"][1], Tw["Wg"][0], Tw["Wu"][1], Tw["Wu"][0], Tw["Wd"][1],
            Tw["Wd"][0], eps=1e-5)), per_case_s)
        full = dt * d["M"] / rows
        out["ffn"] = {"us": full * 1e6,
                      "TOPS": (2 * 2 * d["M"] * d["H"] * d["I"] + 2 * d["M"] * d["I"] * d["H"])
                      / full / 1e12, "cores": prev, "kind": "oracle",
                      "sample": f"{rows} of {d['M']} tokens, scaled to the full block"}
    finally:
        oracle.set_threads(prev)
    return out


def run_reference(args, world, rank):
    """Reference arm: the CPU oracle as it stands, on this host's cores."""
    if rank != 0:
        return 0
    per_step = args.ref_step_seconds or max(0.5, min(4.0, 150.0 / max(1, args.steps + args.warmup)))
    import oracle
    threads = oracle.num_threads()
    prepared = []
    for i, (K, N) in enumerate(PREFILL_KN):
        inp = synthetic.linear_inputs(PREFILL_M, K, N, seed=i)
        g, T, _ = oracle.quantize_weights(inp["W"])
        prepared.append((K, N, inp["X"], T, g))

    def step(tokens, off):
        for K, N, X, T, g in prepared:
            rows = X[off:off + tokens]
            oracle.round_bf16(oracle.bitlinear(rows, T, g, oracle.PRELUDE_RMSNORM, eps=1e-5))

    t0 = time.perf_counter()
    step(2, 0)
    dt = time.perf_counter() - t0
    tokens = int(max(1, min(PREFILL_M, 2 * per_step / max(dt, 1e-4))))
    for i in range(args.warmup):
        step(tokens, (i * tokens) % (PREFILL_M - tokens + 1))
    times = []
    for i in range(args.steps):
        t0 = time.perf_counter()
        step(tokens, (i * tokens) % (PREFILL_M - tokens + 1))
        times.append(time.perf_counter() - t0)
    total = sum(times)
    ops = sum(2 * tokens * N * K for K, N in PREFILL_KN) * args.steps
    value = ops / total / 1e12
    sample = (f"{tokens} tokens of the {PREFILL_M}-token prefill step per step (both projections,"
              f" RMSNorm + quant + contraction + dequant + bf16 round)")
    line = {"metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": f"prefill BitLinear M={PREFILL_M}, (K,N)=(2560,6912)+(6912,2560)"
                                   ", RMSNorm prelude, bf16 out", "parallelism": "host cores"},
            "cpu_baseline": {"value": value, "unit": "TOPS", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------ GPU timing

class Prefill:
    """Device buffers and the launch sequence of one prefill step."""

    def __init__(self, torch, bn, device):
        self.torch, self.bn = torch, bn
        self.shapes = []
        for i, (K, N) in enumerate(PREFILL_KN):
            inp = synthetic.linear_inputs(PREFILL_M, K, N, seed=i)
            W = torch.from_numpy(inp["W"]).to(device)
            P, g, ws = bn.alloc_packed(N, K, device)
            bn.bitnet_pack_weights(W, P, g, ws)
            del W
            X = torch.from_numpy(inp["X"]).to(device)
            q, s, rs = bn.alloc_quant(PREFILL_M, K, device)
            Y = torch.empty((PREFILL_M, N), dtype=torch.bfloat16, device=device)
            self.shapes.append({"K": K, "N": N, "X": X, "P": P, "g": g, "q": q, "s": s,
                                "rs": rs, "Y": Y, "X_host": None, "Y_host": None})
        torch.cuda.synchronize()
        self.launches_per_step = 2 * len(self.shapes)
        self.copy_in = self.copy_out = None

    def step(self, gemm_events=None):
        bn = self.bn
        for i, sh in enumerate(self.shapes):
            bn.bitnet_quant_act(sh["X"], sh["q"], sh["s"], sh["rs"],
                                prelude=bn.BITNET_PRELUDE_RMSNORM, eps=1e-5)
            if gemm_events is not None:
                gemm_events[i][0].record()
            # the weights are constant: the GEMM may load its first weight tiles
            # while the quantiser runs
            bn.bitnet_linear(sh["q"], sh["s"], sh["rs"], sh["P"], sh["g"], sh["K"], sh["Y"],
                             epilogue=bn.BITNET_BF16 | bn.BITNET_LAUNCH_PDL)
            if gemm_events is not None:
                gemm_events[i][1].record()

    def e2e_buffers(self):
        torch = self.torch
        for sh in self.shapes:
            if sh["X_host"] is None:
                sh["X_host"] = sh["X"].cpu().pin_memory()
                sh["Y_host"] = torch.empty(sh["Y"].shape, dtype=sh["Y"].dtype).pin_memory()
        if self.copy_in is None:
            self.copy_in, self.copy_out = torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_step(self):
        """One step through the public API from and to pinned host buffers,
        pipelined over token chunks: the host-to-device copy of a chunk (copy-in
        stream), its quantiser and projection (the current stream) and the
        device-to-host copy of its outputs (copy-out stream) overlap those of
        the neighbouring chunks, and PCIe carries both directions at once.  The
        step starts after all earlier work on the current stream and ends, on
        that stream, when the last outputs are on the host."""
        torch, bn = self.torch, self.bn
        main = torch.cuda.current_stream()
        self.copy_in.wait_stream(main)
        self.copy_out.wait_stream(main)
        rows = PREFILL_M // E2E_CHUNKS
        for sh in self.shapes:
            for c in range(E2E_CHUNKS):
                sl = slice(c * rows, (c + 1) * rows)
                with torch.cuda.stream(self.copy_in):
                    sh["X"][sl].copy_(sh["X_host"][sl], non_blocking=True)
                landed = torch.cuda.Event()
                landed.record(self.copy_in)
                main.wait_event(landed)
                bn.bitnet_quant_act(sh["X"][sl], sh["q"][sl], sh["s"][sl], sh["rs"][sl],
                                    prelude=bn.BITNET_PRELUDE_RMSNORM, eps=1e-5)
                bn.bitnet_linear(sh["q"][sl], sh["s"][sl], sh["rs"][sl], sh["P"], sh["g"],
                                 sh["K"], sh["Y"][sl], epilogue=bn.BITNET_BF16 | bn.BITNET_LAUNCH_PDL)
                done = torch.cuda.Event()
                done.record(main)
                self.copy_out.wait_event(done)
                with torch.cuda.stream(self.copy_out):
                    sh["Y_host"][sl].copy_(sh["Y"][sl], non_blocking=True)
        main.wait_stream(self.copy_out)

    def h2d_bytes(self):
        return sum(sh["X"].numel() * sh["X"].element_size() for sh in self.shapes)

    def d2h_bytes(self):
        return sum(sh["Y"].numel() * sh["Y"].element_size() for sh in self.shapes)


def time_loop(torch, fn, steps):
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(steps):
        fn()
    end.record()
    end.synchronize()
    return start.elapsed_time(end) / 1e3


def bench_decode(torch, bn, device, reps=3):
    """Steady-state decode GEMV streaming: a CUDA graph of back-to-back calls
    over a pool of distinct packed-weight copies larger than twice the L2, all
    reading one set of activation codes.  Two launch modes: the calls as the
    independent projections they are here (BITNET_LAUNCH_PDL_INPUTS: only the
    output stores wait for the preceding call), and as a dependent chain
    (BITNET_LAUNCH_PDL: activation loads also wait)."""
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    out = []
    modes = (("independent", bn.BITNET_LAUNCH_PDL_INPUTS), ("dependent", bn.BITNET_LAUNCH_PDL))
    for (K, N) in DECODE_KN:
        inp = synthetic.linear_inputs(max(DECODE_M), K, N, seed=K + N)
        W = torch.from_numpy(inp["W"]).to(device)
        P0, g, ws = bn.alloc_packed(N, K, device)
        bn.bitnet_pack_weights(W, P0, g, ws)
        del W
        wbytes = P0.numel()
        pool = max(8, int(2 * l2 // wbytes) + 2)
        pool_bufs = [P0.clone() for _ in range(pool)]
        X = torch.from_numpy(inp["X"]).to(device)
        for M in DECODE_M:
            q, s, rs = bn.alloc_quant(M, K, device)
            bn.bitnet_quant_act(X[:M].contiguous(), q, s, rs)
            Y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
            rec = {"M": M, "K": K, "N": N, "weights_in_pool": pool}
            for name, flag in modes:
                epi = bn.BITNET_BF16 | flag
                for Pb in pool_bufs[:2]:
                    bn.bitnet_linear(q, s, rs, Pb, g, K, Y, epilogue=epi)
                torch.cuda.synchronize()
                graph = torch.cuda.CUDAGraph()
                stream = torch.cuda.Stream(device)
                with torch.cuda.stream(stream):
                    graph.capture_begin(capture_error_mode="thread_local")
                    for Pb in pool_bufs:
                        bn.bitnet_linear(q, s, rs, Pb, g, K, Y, epilogue=epi, stream=stream)
                    graph.capture_end()
                torch.cuda.synchronize()
                graph.replay()
                torch.cuda.synchronize()
                best = None
                for _ in range(reps):
                    dt = time_loop(torch, graph.replay, 4)
                    best = dt if best is None else min(best, dt)
                calls = 4 * pool
                key = "" if name == "independent" else "_dependent"
                rec["us_per_call" + key] = best / calls * 1e6
                rec["GB_s" + key] = decode_bytes(M, K, N) * calls / best / 1e9
                del graph
            out.append(rec)
        del pool_bufs
        torch.cuda.empty_cache()
    return out


QKV_N = (2560, 640, 640)          # q, k, v projections of the 2B model (K = 2560)


def bench_decode_qkv(torch, bn, device, reps=3):
    """The q, k and v decode projections of one input: one bitnet_linear_multi
    call per step (one launch) against three bitnet_linear calls, both as
    independent projections in a CUDA graph over a pool of weight sets larger
    than twice the L2."""
    K = 2560
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    inp = synthetic.linear_inputs(max(DECODE_M), K, sum(QKV_N), seed=11)
    W = torch.from_numpy(inp["W"]).to(device)
    sets, row = [], 0
    base = []
    for N in QKV_N:
        P, g, ws = bn.alloc_packed(N, K, device)
        bn.bitnet_pack_weights(W[row:row + N].contiguous(), P, g, ws)
        base.append((P, g))
        row += N
    del W
    set_bytes = sum(P.numel() for P, _ in base)
    pool = max(8, int(2 * l2 // set_bytes) + 2)
    sets = [[(P.clone(), g) for P, g in base] for _ in range(pool)]
    X = torch.from_numpy(inp["X"]).to(device)
    out = []
    for M in DECODE_M:
        q, s, rs = bn.alloc_quant(M, K, device)
        bn.bitnet_quant_act(X[:M].contiguous(), q, s, rs)
        Ys = [torch.empty((M, N), dtype=torch.bfloat16, device=device) for N in QKV_N]
        epi = bn.BITNET_BF16 | bn.BITNET_LAUNCH_PDL_INPUTS
        bytes_step = sum(decode_bytes(M, K, N) for N in QKV_N)

        def fused(st, ws_):
            bn.bitnet_linear_multi(q, s, rs, [P for P, _ in ws_], [g for _, g in ws_], K, Ys,
                                   epilogue=epi, stream=st)

        def separate(st, ws_):
            for (P, g), Y in zip(ws_, Ys):
                bn.bitnet_linear(q, s, rs, P, g, K, Y, epilogue=epi, stream=st)
        rec = {"M": M, "K": K, "N": list(QKV_N), "weight_sets_in_pool": pool}
        for name, fn in (("fused", fused), ("separate", separate)):
            fn(None, sets[0])
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            stream = torch.cuda.Stream(device)
            with torch.cuda.stream(stream):
                graph.capture_begin(capture_error_mode="thread_local")
                for ws_ in sets:
                    fn(stream, ws_)
                graph.capture_end()
            torch.cuda.synchronize()
            graph.replay()
            torch.cuda.synchronize()
            best = min(time_loop(torch, graph.replay, 4) for _ in range(reps))
            rec["us_per_step_" + name] = best / (4 * pool) * 1e6
            rec["GB_s_" + name] = bytes_step * 4 * pool / best / 1e9
            del graph
        out.append(rec)
    del sets
    torch.cuda.empty_cache()
    return out


def bench_ffn(torch, bn, device, iters=20):
    cfg = synthetic.WORKLOADS["ffn"].dims
    M, H, I = cfg["M"], cfg["H"], cfg["I"]
    inp = synthetic.ffn_inputs(M, H, I, seed=0)
    packs = []
    for k in ("Wg", "Wu", "Wd"):
        W = torch.from_numpy(inp[k]).to(device)
        P, g, ws = bn.alloc_packed(*W.shape, device)
        bn.bitnet_pack_weights(W, P, g, ws)
        packs.append((P, g))
    X = torch.from_numpy(inp["x_bf16"].view(np.int16)).to(device).view(torch.bfloat16)
    Y = torch.empty((M, H), dtype=torch.bfloat16, device=device)
    ws = bn.alloc_ffn_workspace(M, H, I, device=device)

    def run():
        bn.bitnet_ffn(X, packs[0][0], packs[0][1], packs[1][0], packs[1][1], packs[2][0],
                      packs[2][1], Y, ws, variant=bn.BITNET_FFN_RELU2_GLU, eps=1e-5)
    for _ in range(3):
        run()
    dt = time_loop(torch, run, iters) / iters
    ops = 2 * 2 * M * H * I + 2 * M * I * H
    return {"M": M, "H": H, "I": I, "us": dt * 1e6, "TOPS": ops / dt / 1e12}


def bench_decode_ffn(torch, bn, device, reps=3):
    """The W1.58A8 block FFN at decode sizes (M = 1, 4, 16 tokens of the
    2560 -> 6912 -> 2560 FFN): back-to-back bitnet_ffn calls in a CUDA graph
    over a pool of weight sets larger than twice the L2, as the default
    four-launch route (quant, gate + up, relu^2 * up with the sub-norm quant,
    down) and as one persistent launch per FFN (BITNET_FFN_SINGLE_LAUNCH).  GB/s counts the three packed
    weight matrices, x (read twice) and y."""
    cfg = synthetic.WORKLOADS["ffn"].dims
    H, I = cfg["H"], cfg["I"]
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    inp = synthetic.ffn_inputs(max(DECODE_M), H, I, seed=5)
    base = []
    for k in ("Wg", "Wu", "Wd"):
        W = torch.from_numpy(inp[k]).to(device)
        P, g, ws = bn.alloc_packed(*W.shape, device)
        bn.bitnet_pack_weights(W, P, g, ws)
        base.append((P, g))
    set_bytes = sum(P.numel() for P, _ in base)
    pool = max(8, int(2 * l2 // set_bytes) + 2)
    sets = [[(P.clone(), g) for P, g in base] for _ in range(pool)]
    X_all = torch.from_numpy(inp["x_bf16"].view(np.int16)).to(device).view(torch.bfloat16)
    out = []
    for M in DECODE_M:
        X = X_all[:M].contiguous()
        Y = torch.empty((M, H), dtype=torch.bfloat16, device=device)
        ws = bn.alloc_ffn_workspace(M, H, I, device=device)
        step_bytes = set_bytes + 3 * 2 * M * H      # + x (twice: norm, residual) and y, bf16

        rec = {"M": M, "H": H, "I": I, "weight_sets_in_pool": pool}
        # one persistent launch per FFN (the default), and the four-launch route
        for key, variant in (("", bn.BITNET_FFN_RELU2_GLU),
                             ("_single_launch",
                              bn.BITNET_FFN_RELU2_GLU | bn.BITNET_FFN_SINGLE_LAUNCH)):
            def run(st, w):
                bn.bitnet_ffn(X, w[0][0], w[0][1], w[1][0], w[1][1], w[2][0], w[2][1], Y, ws,
                              variant=variant, eps=1e-5, stream=st)
            run(None, sets[0])
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            stream = torch.cuda.Stream(device)
            with torch.cuda.stream(stream):
                graph.capture_begin(capture_error_mode="thread_local")
                for w in sets:
                    run(stream, w)
                graph.capture_end()
            torch.cuda.synchronize()
            graph.replay()
            torch.cuda.synchronize()
            best = min(time_loop(torch, graph.replay, 4) for _ in range(reps))
            rec["us_per_ffn" + key] = best / (4 * pool) * 1e6
            rec["GB_s" + key] = step_bytes * 4 * pool / best / 1e9
            del graph
        out.append(rec)
    del sets
    return out


def bench_hffn(torch, bn, device, iters=50):
    cfg = synthetic.WORKLOADS["hffn"].dims
    M, D, F = cfg["M"], cfg["D"], cfg["F"]
    inp = synthetic.hffn_inputs(M, D, F, seed=0)
    packs = []
    for k in ("W1", "W2"):
        W = torch.from_numpy(inp[k]).to(device)
        P, g, ws = bn.alloc_packed(*W.shape, device)
        bn.bitnet_pack_weights(W, P, g, ws)
        packs.append((P, g))
    X = torch.from_numpy(inp["X"]).to(device)
    Y = torch.empty((M, D), device=device)
    ws = bn.alloc_ffn_workspace(M, D, F, bn.BITNET_FFN_HADAMARD_SILU, device=device)

    def run():
        bn.bitnet_ffn(X, packs[0][0], packs[0][1], None, None, packs[1][0], packs[1][1], Y, ws,
                      variant=bn.BITNET_FFN_HADAMARD_SILU)
    for _ in range(3):
        run()
    dt = time_loop(torch, run, iters) / iters
    ops = 2 * 2 * M * D * F
    return {"M": M, "D": D, "F": F, "us": dt * 1e6, "TOPS": ops / dt / 1e12}


def bench_tiny(torch, bn, device, iters=200):
    d = synthetic.WORKLOADS["tiny"].dims
    M, K, N = d["M"], d["K"], d["N"]
    inp = synthetic.linear_inputs(M, K, N, seed=0)
    W = torch.from_numpy(inp["W"]).to(device)
    P, g, ws = bn.alloc_packed(N, K, device)
    bn.bitnet_pack_weights(W, P, g, ws)
    X = torch.from_numpy(inp["X"]).to(device)
    q, s, rs = bn.alloc_quant(M, K, device)
    Y = torch.empty((M, N), device=device)

    def run(stream=None):
        bn.bitnet_quant_act(X, q, s, rs, stream=stream)
        bn.bitnet_linear(q, s, rs, P, g, K, Y, epilogue=bn.BITNET_F32 | bn.BITNET_LAUNCH_PDL,
                         stream=stream)
    for _ in range(5):
        run()
    dt = time_loop(torch, run, iters) / iters
    # the same pairs replayed from a CUDA graph: device time without the
    # Python and launch overhead of each call
    reps = 20
    graph = torch.cuda.CUDAGraph()
    stream = torch.cuda.Stream(device)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        graph.capture_begin(capture_error_mode="thread_local")
        for _ in range(reps):
            run(stream)
        graph.capture_end()
    torch.cuda.synchronize()
    graph.replay()
    torch.cuda.synchronize()
    dg = min(time_loop(torch, graph.replay, 10) for _ in range(3)) / (10 * reps)
    del graph
    return {"M": M, "K": K, "N": N, "us_per_call": dt * 1e6, "us_per_call_graph": dg * 1e6,
            "note": "quant + linear: eager calls are bound by host launch overhead; the graph "
                    "replay gives the device time of a dependent pair"}


def bench_online(torch, bn, device, iters=20):
    """Online ternarisation: the bf16 master weights re-ternarised every
    forward (absmean pass + pack) ahead of the prefill projection, against
    the same projection on stored packed weights.  M = 4096, K = 2560,
    N = 6912, RMSNorm prelude, bf16 out."""
    M, K, N = PREFILL_M, 2560, 6912
    inp = synthetic.linear_inputs(M, K, N, seed=0)
    Wb = torch.from_numpy(inp["W"]).to(device).to(torch.bfloat16)
    X = torch.from_numpy(inp["X"]).to(device)
    P, g, ws = bn.alloc_packed(N, K, device)
    q, s, rs = bn.alloc_quant(M, K, device)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=device)

    def pack():
        bn.bitnet_pack_weights(Wb, P, g, ws)

    def project():
        bn.bitnet_quant_act(X, q, s, rs, prelude=bn.BITNET_PRELUDE_RMSNORM, eps=1e-5)
        bn.bitnet_linear(q, s, rs, P, g, K, Y)

    def online():
        pack()
        project()
    out = {"M": M, "K": K, "N": N, "weights": "bf16 master copy, re-packed per forward"}
    for name, fn in (("pack_us", pack), ("stored_weights_us", project), ("online_us", online)):
        for _ in range(3):
            fn()
        out[name] = time_loop(torch, fn, iters) / iters * 1e6
    return out


def run_b200(args, world, rank, local):
    import torch
    if not torch.cuda.is_available():
        print(json.dumps({"metric": METRIC, "error": "no CUDA device"}), flush=True)
        return 1
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    import ternary_weight_token_b200 as bn
    bn.library()
    peaks = measured_peaks()

    pre = Prefill(torch, bn, device)
    # the clock sampler starts before the warm-up steps, so the timed steps
    # follow the warm-up directly (no idle GPU in between)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.15)
    for _ in range(max(3, args.warmup)):
        pre.step()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()

    # ---- timed region: K steps as a user runs them (no events between the
    # kernels: an event recorded between two launches stops the second from
    # starting under the first with programmatic dependent launch, which cost
    # ~11 us per step); then the same K steps again with every GEMM launch
    # bracketed by CUDA events on the stream it is launched on (torch's
    # current stream), for the GEMM's per-launch duration
    n_sh = len(pre.shapes)
    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(n_sh)] for _ in range(args.steps)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    t_wall0 = time.time()
    nvtx_push(torch, f"prefill: {args.steps} timed steps")
    start.record()
    for s in range(args.steps):
        pre.step()
    end.record()
    nvtx_pop(torch)
    end.synchronize()
    elapsed = start.elapsed_time(end) / 1e3
    nvtx_push(torch, f"prefill: {args.steps} steps with per-GEMM events")
    for s in range(args.steps):
        pre.step(evs[s])
    torch.cuda.synchronize()
    nvtx_pop(torch)
    t_wall1 = time.time()
    clocks = sampler.stop((t_wall0, t_wall1))
    gemm_avg = [sum(evs[s][i][0].elapsed_time(evs[s][i][1]) for s in range(args.steps))
                / args.steps / 1e3 for i in range(n_sh)]
    if dist is not None:
        dist.barrier()
    elapsed = max_over_ranks(elapsed, dist, device)

    ms_per_step = elapsed / args.steps * 1e3
    value = world * prefill_ops() * args.steps / elapsed / 1e12

    # ---- e2e through the C ABI with host buffers
    pre.e2e_buffers()
    e2e_steps = max(3, min(args.steps, 20))
    for _ in range(2):
        pre.e2e_step()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    nvtx_push(torch, f"prefill e2e: {e2e_steps} steps from host buffers")
    e2e_elapsed = time_loop(torch, pre.e2e_step, e2e_steps)
    nvtx_pop(torch)
    e2e_elapsed = max_over_ranks(e2e_elapsed, dist, device)
    e2e_value = world * prefill_ops() * e2e_steps / e2e_elapsed / 1e12

    # ---- roofline of the dominant kernel (tcgen05 GEMM)
    int8_peak = 2.0 * peaks["bf16_tflops"]
    gemm_ops = [2 * PREFILL_M * N * K for K, N in PREFILL_KN]
    achieved = sum(gemm_ops) / sum(gemm_avg) / 1e12
    traffic = profiled_traffic()
    roofline = {"bound": "tensor", "achieved": achieved, "peak": int8_peak, "unit": "TOP/s",
                "frac": achieved / int8_peak, "traffic": traffic,
                "kernel": "gemm_tc_kernel (tcgen05.mma kind::i8)",
                "peak_source": f"{peaks['source']} bf16 burst {peaks['bf16_tflops']} TF/s x 2 "
                               "(int8/bf16 nominal ratio 4.5/2.25)",
                "per_launch_us": [t * 1e6 for t in gemm_avg],
                "ops_per_launch": gemm_ops,
                "timing": "CUDA events around each GEMM launch over K steps run right after "
                          "the K timed steps (which carry no events between kernels)"}

    line = {"metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "int8", "data": "synthetic",
            "config": {"workload": f"prefill BitLinear M={PREFILL_M} tokens per GPU, (K,N)="
                                   "(2560,6912)+(6912,2560), RMSNorm prelude + per-token int8 "
                                   "quant + ternary contraction + bf16 dequant",
                       "M": PREFILL_M, "shapes": [list(s) for s in PREFILL_KN],
                       "l2": "inputs larger than L2: 155 MB of fp32 activations and 113 MB of "
                             "bf16 outputs per step",
                       "parallelism": f"dp{world} (tokens sharded, no data-path collective)"},
            "roofline": roofline,
            "e2e": {"value": e2e_value, "unit": "TOPS",
                    "h2d_bytes_per_step": pre.h2d_bytes(),
                    "d2h_bytes_per_step": pre.d2h_bytes(), "steps": e2e_steps},
            "gpu_launches": pre.launches_per_step * args.steps,
            "clocks": clocks,
            "source": {"csrc_sha256_16": sources_sha()}}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_prefill_sample(target_s=args.cpu_seconds)
    if rank == 0 and not args.no_extra:
        dec = bench_decode(torch, bn, device)
        for d in dec:
            d["frac_of_hbm"] = d["GB_s"] / peaks["hbm_gbs"]
            d["frac_of_hbm_dependent"] = d["GB_s_dependent"] / peaks["hbm_gbs"]
        def extra(fn):
            # a failing secondary workload is reported in its slot; the
            # headline line is printed regardless
            try:
                return fn(torch, bn, device)
            except Exception as e:        # noqa: BLE001
                return {"error": f"{type(e).__name__}: {e}"}
        line["workloads"] = {
            "decode": dec,
            "decode_qkv": extra(bench_decode_qkv),
            "decode_ffn": extra(bench_decode_ffn),
            "decode_peak_source": f"{peaks['source']} HBM copy {peaks['hbm_gbs']} GB/s",
            "ffn": extra(bench_ffn),
            "hffn": extra(bench_hffn),
            "tiny": extra(bench_tiny),
            "online_ternarisation": extra(bench_online),
        }
        if not args.no_cpu_baseline:
            # the oracle beside every secondary workload (same inputs)
            try:
                base = oracle_workload_baselines()
                w = line["workloads"]
                for name in ("tiny", "hffn", "ffn"):
                    if isinstance(w.get(name), dict):
                        w[name]["cpu_baseline"] = base[name]
                for rec in w["decode"]:
                    for b in base["decode"]:
                        if (b["M"], b["K"], b["N"]) == (rec["M"], rec["K"], rec["N"]):
                            rec["cpu_baseline"] = b
            except Exception as e:        # noqa: BLE001
                line["workloads"]["cpu_baseline_error"] = f"{type(e).__name__}: {e}"
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def decode_single(torch, bn, device, M, K, N, iters, independent=False):
    """Plain back-to-back launches of one decode shape (no graph): the short
    command the decode kernel is profiled with (independent: the calls carry
    BITNET_LAUNCH_PDL_INPUTS, as independent projections do)."""
    inp = synthetic.linear_inputs(M, K, N, seed=K + N)
    W = torch.from_numpy(inp["W"]).to(device)
    P, g, ws = bn.alloc_packed(N, K, device)
    bn.bitnet_pack_weights(W, P, g, ws)
    X = torch.from_numpy(inp["X"]).to(device)
    q, s, rs = bn.alloc_quant(M, K, device)
    bn.bitnet_quant_act(X, q, s, rs)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=device)

    epi = bn.BITNET_BF16 | (bn.BITNET_LAUNCH_PDL_INPUTS if independent else 0)

    def run():
        bn.bitnet_linear(q, s, rs, P, g, K, Y, epilogue=epi)
    for _ in range(3):
        run()
    dt = time_loop(torch, run, iters) / iters
    return {"M": M, "K": K, "N": N, "independent": independent, "us_per_call": dt * 1e6,
            "GB_s": decode_bytes(M, K, N) / dt / 1e9}


def run_only(args, local):
    import torch
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    import ternary_weight_token_b200 as bn
    if args.only == "decode" and args.decode_shape:
        fields = args.decode_shape.split(",")
        M, K, N = (int(v) for v in fields[:3])
        out = decode_single(torch, bn, device, M, K, N, max(1, args.steps),
                            independent=len(fields) > 3 and fields[3] == "independent")
    else:
        fn = {"decode": bench_decode, "ffn": bench_ffn, "hffn": bench_hffn,
              "tiny": bench_tiny, "qkv": bench_decode_qkv, "online": bench_online,
              "dffn": bench_decode_ffn}[args.only]
        out = fn(torch, bn, device)
    print(json.dumps({"only": args.only, "result": out}), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("b200", "reference"), default="b200")
    ap.add_argument("--no-extra", action="store_true", help="skip decode / FFN / tiny workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-step-seconds", type=float, default=None,
                    help="with --impl reference: target seconds of oracle work per step")
    ap.add_argument("--only", choices=("decode", "ffn", "hffn", "tiny", "qkv", "online", "dffn"),
                    default=None,
                    help="time one secondary workload and print its JSON (profiling aid)")
    ap.add_argument("--decode-shape", default=None,
                    help="with --only decode: one 'M,K,N[,independent]' case, no CUDA graph")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_env()
    if args.gpus != world and not (world == 1 and args.gpus == 1):
        if world == 1:
            print(json.dumps({"metric": METRIC, "error": f"--gpus {args.gpus} needs torchrun "
                              f"with {args.gpus} processes"}), flush=True)
            return 2
    if args.impl == "reference":
        return run_reference(args, world, rank)
    if args.only is not None:
        return run_only(args, local)
    return run_b200(args, world, rank, local)


if __name__ == "__main__":
    sys.exit(main())
