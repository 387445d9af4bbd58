#!/usr/bin/env python
"""Throughput of the OFT + dequant linear hot path on B200.

A step is one pass of the whole path over one batch: Cayley build of every
rotation block, the split-projection forward (rotate, dequant, tcgen05 GEMM),
and for the training workloads the adapter backward (dX' GEMM, dX rotation,
dR reduction, Cayley backward), plus the dQ all-reduce when several ranks run
data-parallel replicas.  The headline workload (default) is the largest one that
fits one GPU: the MXFP4 training step, forward + backward (16384 tokens x 7168 ->
12288/3072/3072, b = 64).  On one GPU the other four workloads are timed after it
(--also) and reported in the same line under "workloads".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c4] [--also c0,c1,c2,c3]
                    [--impl ours|reference]

With --gpus N > 1 and no WORLD_SIZE in the environment, the script starts N ranks
itself (torch.distributed.run, one process per GPU).  Prints one JSON line (rank 0).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "OFT+dequant linear fwd/bwd tokens/s, TFLOP/s vs B200 dense tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20

WORKLOAD_NAMES = {
    "c0": "tiny fused-QKV OFT linear fwd: 64 x 256 -> 3x128, INT4 g32, b=32",
    "c1": "dense fused-QKV OFT linear fwd+bwd: 4096 x 2560 -> 4096/1024/1024, FP8 e4m3 per-channel, b=32",
    "c2": "gated-MLP gate/up OFT linear fwd: 8192 x 4096 -> 2x12288, INT4 g128, b=64",
    "c3": "MoE active-expert-chunked OFT fwd: 4096 tok, hidden 7168, 384 experts x (2x2048), INT4 g32, top-8, chunk 16, b=32",
    "c4": "training-step OFT linear fwd+bwd: 16384 x 7168 -> 12288/3072/3072, MXFP4, b=64",
    # decode-like checks, not among the five workloads: the same weights at 64 tokens, forward only
    "c1-m64": "fused-QKV FP8 weights at 64 tokens, fwd: 64 x 2560 -> 4096/1024/1024, FP8 e4m3 per-channel, b=32",
    "c4-m64": "MXFP4 weights at 64 tokens, fwd: 64 x 7168 -> 12288/3072/3072, MXFP4, b=64",
    # a smaller MoE case for profiler captures (the full layer holds ~12 GB): same expert shapes
    "c3-mid": "MoE active-expert-chunked OFT: 2048 tok, hidden 7168, 128 experts x (2x2048), INT4 g32, top-8, chunk 16, b=32",
}


def moe_spec(name: str):
    from gen import MOE_CONFIGS
    if name == "c3-mid":
        return MOE_CONFIGS["c3"].with_(name="c3-mid", T=2048, E=128)
    return MOE_CONFIGS.get(name)


def linear_spec(name: str):
    """The linear workload `name`: one of the five, or a 64-token forward over c1 / c4 weights."""
    from gen import LINEAR_CONFIGS
    if name.endswith("-m64"):
        return LINEAR_CONFIGS[name[:-4]].with_(M=64, backward=False)
    return LINEAR_CONFIGS[name]


# ----------------------------------------------------------------------------
# helpers (also used by the multi-process CPU tests)
# ----------------------------------------------------------------------------

def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def init_dist(backend: str):
    import datetime
    import torch.distributed as dist
    rank, world, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world


def max_over_ranks(x: float, device) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def allreduce_grad(dQ):
    """Data-parallel replicas: sum the adapter gradient over ranks (the only
    exchange the path has; the frozen base has no gradient)."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(dQ)
    return dQ


def token_shard(M: int, rank: int, world: int):
    """Contiguous token range [t0, t1) of `rank` when one batch of M tokens is split
    over `world` data-parallel replicas (the first M % world ranks take one more)."""
    base, extra = divmod(M, world)
    t0 = rank * base + min(rank, extra)
    return t0, t0 + base + (1 if rank < extra else 0)


def launch_cmd(argv, nproc: int, port: int, limit_s: int = 3600):
    """The command that runs this script as `nproc` ranks on one node (one process
    per GPU), bounded by `timeout`."""
    return ["timeout", "-k", "60", str(limit_s), sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={nproc}", "--master-addr", "127.0.0.1", f"--master-port={port}",
            os.path.abspath(__file__), *argv]


def workload_config(name: str, tokens: int, world: int, backward: bool, args, n_active=None):
    """The `config` object of a line: the same for our arm and the reference arm."""
    config = {"workload": WORKLOAD_NAMES[name], "name": name, "tokens_per_gpu": tokens,
              "global_batch_tokens": tokens * world, "parallelism": f"dp{world}" if world > 1 else "single",
              "l2": f"flushed between timed steps ({L2_FLUSH_BYTES >> 20} MB write)",
              "step": "build_rotation + fwd" + (" + bwd" if backward else "")
                      + (" + dQ all-reduce" if world > 1 and backward else "")}
    if moe_spec(name) is not None:
        config.update(n_active_experts=n_active, moe_variant=args.moe)
        config["step"] = ("route + build_rotation + fwd" + (" + bwd (dX, dQ, dlogits)" if backward else "")
                          + (" (full expert layer: gate/up, SwiGLU, down)" if args.moe_layer else ""))
    elif args.weight_side:
        config["variant"] = "weight-side rotation: Y_p = X (R_p deq(W_p))"
    return config


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def linear_flops(spec, backward: bool):
    M, K, N, P, b = spec.M, spec.K, spec.N, spec.P, spec.b
    nblk = P * (K // b)
    gemm = 2.0 * M * K * N
    rot = 2.0 * M * K * b * P
    f = dict(gemm_fwd=gemm, rot_fwd=rot, cayley=2.0 * b ** 3 * nblk)
    if backward:
        f.update(gemm_bwd=gemm, rot_dx=rot, rot_dr=rot, cayley_bwd=4.0 * b ** 3 * nblk)
    return f


def weight_bytes(spec):
    N, K = spec.N, spec.K
    if spec.fmt == "fp8":
        return N * K + 4 * N
    if spec.fmt == "int4":
        return N * K // 2 + 2 * N * (K // spec.group)
    return N * K // 2 + N * (K // 32)


# ----------------------------------------------------------------------------
# clocks (NVML, sampled in a thread during the timed region)
# ----------------------------------------------------------------------------

_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
            0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
            0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


def tensor_peak(peaks, clk):
    """The measured bf16 peak that matches the clocks seen in the timed region: the
    sustained figure (taken under the power cap) when the power cap was active or the
    SM clock sat below 95 % of its maximum, else the burst figure (full clock).  With no
    clock record the burst figure, the larger of the two."""
    reasons = clk.get("reasons") or []
    mhz, top = clk.get("sm_mhz"), clk.get("sm_max_mhz")
    capped = "sw_power_cap" in reasons or (mhz is not None and top and mhz < 0.95 * top)
    if capped and "bf16_tflops_sustained" in peaks:
        return peaks["bf16_tflops_sustained"], "sustained"
    return peaks["bf16_tflops"], "burst"


class ClockSampler:
    def __init__(self, torch_device, period_s: float = 0.02):
        self.samples, self.reasons, self.power = [], set(), []
        self.max_mhz = None
        self.period = period_s
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(torch_device).uuid)
            try:
                self._h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-") else uuid)
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(torch_device.index or 0)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._nvml = pynvml
        except Exception as e:  # no NVML: report no samples
            self.error = repr(e)
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in _REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
                self.power.append(nv.nvmlDeviceGetPowerUsage(self._h) / 1000.0)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._h is not None:
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._h is not None:
            self._t.join()
        return False

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples),
                "power_w_max": max(self.power) if self.power else None}


# ----------------------------------------------------------------------------
# the oracle as a CPU baseline
# ----------------------------------------------------------------------------

def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 0) for d in threadpool_info() if d.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return "unknown"


def oracle_linear_step(case, tokens: int, backward: bool):
    """One oracle step (float64, numpy) on the first `tokens` tokens: dequant the
    frozen weight, Cayley build, forward, and the adapter backward."""
    import numpy as np
    from oracle import oft_ref
    from oracle.codecs import bf16_bits_to_f64
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from npcase import linear_np
    c = linear_np(case)
    spec = case["spec"]
    t0 = time.perf_counter()
    Wt = oft_ref.weight_t(c)
    R = oft_ref.rotations(c["Q"], spec.b)
    X = bf16_bits_to_f64(c["X"][:tokens])
    oft_ref.linear_fwd(X, Wt, spec.splits, R)
    if backward:
        dY = bf16_bits_to_f64(c["dY"][:tokens])
        oft_ref.linear_bwd(dY, X, Wt, spec.splits, R, spec.b)
    return time.perf_counter() - t0


def cpu_baseline_linear(case, backward: bool, budget_s: float = 12.0):
    spec = case["spec"]
    tokens = min(spec.M, 128)
    dt = oracle_linear_step(case, tokens, backward)
    while dt < budget_s / 3 and tokens < spec.M:
        tokens = min(spec.M, tokens * 4)
        dt = oracle_linear_step(case, tokens, backward)
    return {"value": tokens / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"first {tokens} of {spec.M} tokens, whole weight dequantised, float64 numpy "
                      f"({cpu_model()}), {dt:.2f} s"}


def cpu_baseline_moe(case, budget_s: float = 12.0, dY=None, down=None):
    """Oracle tokens/s of the MoE step on the host cores (forward; with dY, forward +
    backward; with the down projections, the full expert layer)."""
    import numpy as np
    from oracle import moe_ref
    from oracle.codecs import bf16_bits_to_f64
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from npcase import raw
    spec = case["spec"]
    dYf = None if dY is None else bf16_bits_to_f64(raw(dY[:8]))
    logits = raw(case["logits"])
    idx, _ = moe_ref.topk(logits, spec.top_k)
    t0 = time.perf_counter()
    done = 0
    X = raw(case["X"])
    while time.perf_counter() - t0 < budget_s and done < 8:
        t = done
        used = np.unique(idx[t])
        codes = {int(e): raw(case["codes"][int(e)]) for e in used}
        scales = {int(e): raw(case["scales"][int(e)]) for e in used}
        bank = moe_ref.ExpertBank(codes, scales, spec.K, spec.group, spec.n_proj)
        if down is not None:
            dcodes = {int(e): raw(down["down_codes"][int(e)]) for e in used}
            dscales = {int(e): raw(down["down_scales"][int(e)]) for e in used}
            dbank = moe_ref.DownBank(dcodes, dscales, spec.n_proj, spec.group)
            moe_ref.moe_layer_direct(X[t:t + 1], logits[t:t + 1], bank, dbank, raw(case["Q"]), raw(down["Q_down"]),
                                     spec.b, spec.top_k)
        else:
            moe_ref.moe_fwd_direct(X[t:t + 1], logits[t:t + 1], bank, raw(case["Q"]), spec.b, spec.top_k)
        if dYf is not None:
            moe_ref.moe_bwd_direct(dYf[t:t + 1], X[t:t + 1], logits[t:t + 1], bank, raw(case["Q"]), spec.b,
                                   spec.top_k, spec.E)
        done += 1
    dt = time.perf_counter() - t0
    what = ("forward + backward" if dYf is not None else
            "full expert layer" if down is not None else "direct per-token top-%d sum" % spec.top_k)
    return {"value": done / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{done} tokens of {spec.T}, {what}, float64 numpy ({cpu_model()}), {dt:.2f} s"}


# ----------------------------------------------------------------------------
# our path
# ----------------------------------------------------------------------------

# device sources each GEMM kernel is built from (its traffic entry is void once they change)
GEMM_SOURCES = {"gemm_dq2_kernel": ("gemm_dq.cuh", "gemm_dq2.cuh", "dq_pack.cuh"),
                "gemm_bf16_kernel": ("gemm.cuh",), "gemm_bf16_pair_kernel": ("gemm.cuh",)}
PLAIN_MIN_TOKENS = 2048  # the library's switch to the bf16 weight copy + plain GEMM


def gemm_traffic(kernel: str, workload: str):
    """Per-launch DRAM bytes of a GEMM kernel from the committed ncu summary, if the
    kernel's sources are unchanged since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "gemm_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f).get(kernel, {})
    if d.get("kernel_sha256_16") != gemm_kernel_hash(kernel):
        return None
    return d.get("bytes_per_launch_by_workload", {}).get(workload)


def gemm_kernel_hash(kernel: str = "gemm_dq2_kernel") -> str:
    """Hash of a GEMM kernel's device sources."""
    h = hashlib.sha256()
    for f in GEMM_SOURCES[kernel]:
        with open(os.path.join(ROOT, "orthogonal_fine_tuning_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def run_ours(args, rank, world, name):
    import torch
    import orthogonal_fine_tuning_b200 as oft
    from gen import LINEAR_CONFIGS, MOE_CONFIGS, make_linear_case, make_moe_case, make_moe_down, make_moe_grad

    _, _, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    oft.oft_set_gemm_mode(args.gemm_mode)
    peaks, peak_src = load_peaks()
    is_moe = moe_spec(name) is not None
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    if is_moe:
        spec = moe_spec(name)
        case = make_moe_case(spec, device=dev)
        W = oft.Weight("int4", case["codes"], case["scales"], spec.K, 2 * spec.n_proj, spec.group, n_experts=spec.E)
        fused = args.moe == "fused"
        moe_ws = oft.moe_fused_oft_workspace if fused else oft.moe_chunked_oft_workspace
        moe_fwd = oft.moe_fused_oft_fwd if fused else oft.moe_chunked_oft_fwd
        ws = torch.empty(moe_ws(spec.T, spec.E, spec.top_k, spec.chunk, W, spec.b), dtype=torch.uint8, device=dev)
        X, logits, Q = case["X"], case["logits"], case["Q"]
        out = moe_fwd(X, logits, W, spec.b, Q, spec.top_k, spec.chunk, workspace=ws)
        tokens = spec.T
        backward = bool(args.moe_backward)
        if backward:
            # adapter backward through the chunked path: dX, per-expert dQ, router-logit gradient
            dY = make_moe_grad(spec, device=dev)
            bws = torch.empty(oft.moe_chunked_oft_bwd_workspace(spec.T, spec.E, spec.top_k, spec.chunk, W, spec.b),
                              dtype=torch.uint8, device=dev)
            out.update(oft.moe_chunked_oft_bwd(dY, X, logits, W, spec.b, Q, spec.top_k, spec.chunk, workspace=bws))

        def new_outputs():
            o = moe_fwd(X, logits, W, spec.b, Q, spec.top_k, spec.chunk, workspace=ws)
            if backward:
                o.update(oft.moe_chunked_oft_bwd(dY, X, logits, W, spec.b, Q, spec.top_k, spec.chunk, workspace=bws))
            return o

        def step(Xi=X, Li=logits, Qi=Q, o=None, dYi=None):
            o = out if o is None else o
            moe_fwd(Xi, Li, W, spec.b, Qi, spec.top_k, spec.chunk, workspace=ws, out=o)
            if backward:
                oft.moe_chunked_oft_bwd(dY if dYi is None else dYi, Xi, Li, W, spec.b, Qi, spec.top_k, spec.chunk,
                                        workspace=bws, out=o)
                allreduce_grad(o["dQ"])
            return o["Y"]

        inputs = dict(X=X, logits=logits, Q=Q)
        result_keys = ("Y",)
        if backward:
            inputs["dY"] = dY
            result_keys = ("Y", "dX", "dQ", "dlogits")
        if args.moe_layer:
            # full expert layer: gate/up, SwiGLU, down projection with its own adapter
            dn = make_moe_down(spec, device=dev)
            Wd = oft.Weight("int4", dn["down_codes"], dn["down_scales"], spec.n_proj, spec.K, spec.group,
                            n_experts=spec.E)
            Qd = dn["Q_down"]
            lws = torch.empty(oft.moe_chunked_oft_layer_workspace(spec.T, spec.E, spec.top_k, spec.chunk, W, Wd, spec.b),
                              dtype=torch.uint8, device=dev)
            lay = dict(Y=torch.empty(spec.T, spec.K, dtype=torch.bfloat16, device=dev))

            def new_outputs():
                return dict(Y=torch.empty(spec.T, spec.K, dtype=torch.bfloat16, device=dev))

            def step(Xi=X, Li=logits, Qi=Q, o=None, dYi=None, Qdi=None):
                o = lay if o is None else o
                oft.moe_chunked_oft_layer_fwd(Xi, Li, W, Wd, spec.b, Qi, Qd if Qdi is None else Qdi, spec.top_k,
                                              spec.chunk, workspace=lws, out=o["Y"])
                return o["Y"]

            inputs = dict(X=X, logits=logits, Q=Q, Q_down=Qd)
            result_keys = ("Y",)
    else:
        spec = linear_spec(name)
        backward = spec.backward
        case = make_linear_case(spec)
        W = oft.Weight(spec.fmt, case["codes"].to(dev), case["scales"].to(dev), spec.K, spec.N, spec.group)
        X, Q = case["X"].to(dev), case["Q"].to(dev)
        dY = case["dY"].to(dev) if backward else None
        if rank > 0:
            # data-parallel replicas: the same frozen weight and adapter; rank r holds tokens
            # [t0, t1) of a global batch of world x M (weak scaling), drawn from their own seed
            t0, _t1 = token_shard(spec.M * world, rank, world)
            g = torch.Generator(device=dev)
            g.manual_seed(10007 * t0 + spec.seed)
            X = torch.randn(spec.M, spec.K, generator=g, device=dev).to(torch.bfloat16)
            if backward:
                dY = torch.randn(spec.M, spec.N, generator=g, device=dev).to(torch.bfloat16)
        nbytes = oft.oft_linear_fwd_workspace(spec.M, W, spec.splits, spec.b)
        if backward:
            nbytes = max(nbytes, oft.oft_linear_bwd_workspace(spec.M, W, spec.splits, spec.b))
        ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        R = torch.empty(spec.P, spec.K // spec.b, spec.b, spec.b, dtype=torch.float32, device=dev)
        Y = torch.empty(spec.M, spec.N, dtype=torch.bfloat16, device=dev)
        dX = torch.empty(spec.M, spec.K, dtype=torch.bfloat16, device=dev)
        dQ = torch.empty(spec.P, spec.K // spec.b, spec.b * (spec.b - 1) // 2, dtype=torch.float32, device=dev)
        tokens = spec.M

        def new_outputs():
            return dict(Y=torch.empty_like(Y), dX=torch.empty_like(dX), dQ=torch.empty_like(dQ))

        fwd = oft.oft_linear_fwd
        if args.weight_side:
            # the rotation moved onto the weight: Y_p = X (R_p deq(W_p)), one plain bf16 GEMM
            wsw = torch.empty(oft.oft_linear_fwd_weight_side_workspace(W), dtype=torch.uint8, device=dev)

            def fwd(Xi, Wi, splits, b, Ri, Y=None, workspace=None):
                return oft.oft_linear_fwd_weight_side(Xi, Wi, splits, b, Ri, Y=Y, workspace=wsw)

        def step(Xi=X, dYi=dY, Qi=Q, o=None):
            o = dict(Y=Y, dX=dX, dQ=dQ) if o is None else o
            oft.oft_build_rotation(Qi, spec.b, R=R)
            fwd(Xi, W, spec.splits, spec.b, R, Y=o["Y"], workspace=ws)
            if backward:
                oft.oft_linear_bwd(dYi, Xi, W, spec.splits, spec.b, R, dX=o["dX"], dQ=o["dQ"], workspace=ws)
                allreduce_grad(o["dQ"])
            return o["Y"]

        def bwd_part():  # rank-local: the all-reduce is not one of the library calls timed here
            oft.oft_linear_bwd(dY, X, W, spec.splits, spec.b, R, dX=dX, dQ=dQ, workspace=ws)

        # the same step as its API calls, each timed on its own in a third pass
        step_parts = [("build_rotation", lambda: oft.oft_build_rotation(Q, spec.b, R=R)),
                      ("fwd", lambda: fwd(X, W, spec.splits, spec.b, R, Y=Y, workspace=ws))]
        if backward:
            step_parts.append(("bwd", bwd_part))

        inputs = dict(X=X, Q=Q) if not backward else dict(X=X, dY=dY, Q=Q)
        outputs = dict(Y=Y) if not backward else dict(Y=Y, dX=dX, dQ=dQ)
        result_keys = tuple(outputs)

    # ---- device-resident timing ----
    if is_moe:
        step_parts = None
    for _ in range(args.warmup):
        step()
    oft.oft_check_device()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    # Two passes of the same K steps.  The first gives the step time (value): only the
    # step's own launches, so consecutive kernels overlap their launch as they do in use.
    # The second brackets every library kernel with CUDA events on its stream (the
    # library's profiling hooks) for the per-kernel split and the roofline; those events
    # sit between the kernels and add their own gaps, so its step time is reported apart.
    def timed_pass():
        st_, en_ = ([torch.cuda.Event(enable_timing=True) for _ in range(args.steps)] for _ in range(2))
        for i in range(args.steps):
            flush.zero_()                          # evict L2 between timed steps
            st_[i].record()
            step()
            en_[i].record()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        return sum(s.elapsed_time(e) for s, e in zip(st_, en_)) / args.steps

    # The clock sampler runs over every timed pass (the step, the profiled step, the
    # per-call pass and the end-to-end leg) so that short steps still get samples.
    clocks = ClockSampler(dev).__enter__()
    ms_local = timed_pass()
    oft.oft_check_device()
    with oft.profile(max_launches=max(4096, 64 * args.steps)) as prof:
        ms_prof_local = timed_pass()
    oft.oft_check_device()
    # Third pass (dense workloads): CUDA events around each API call of the step, L2
    # flushed before each step.  Rank-local (no collective inside); supplementary: a
    # failure here is reported in the line, and every rank then takes the same
    # max-over-ranks reductions below (a failed part reports -1).
    part_ms = None
    if step_parts is not None:
        part_local, part_err = [-1.0] * len(step_parts), None
        try:
            ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in step_parts]
                  for _ in range(args.steps)]
            for i in range(args.steps):
                flush.zero_()
                for (e0, e1), (_pname, call) in zip(ev[i], step_parts):
                    e0.record()
                    call()
                    e1.record()
            torch.cuda.synchronize()
            for j in range(len(step_parts)):
                part_local[j] = sum(ev[k][j][0].elapsed_time(ev[k][j][1]) for k in range(args.steps)) / args.steps
        except Exception as exc:  # never fatal to the measurement above
            part_err = repr(exc)[:200]
        part_ms = {pname: max_over_ranks(part_local[j], dev) for j, (pname, _c) in enumerate(step_parts)}
        if part_err is not None:
            part_ms["error"] = part_err
        oft.oft_check_device()
    ms_per_step = max_over_ranks(ms_local, dev)
    ms_profiled = max_over_ranks(ms_prof_local, dev)
    value = tokens * world / (ms_per_step / 1e3)

    # ---- algorithmic work ----
    if is_moe:
        n_active = int(out["n_active"].item())
        TK = spec.T * spec.top_k
        gemm_flops = 2.0 * TK * spec.K * 2 * spec.n_proj
        flops = dict(gemm=gemm_flops, rot=2.0 * TK * spec.K * spec.b * 2,
                     cayley=2.0 * spec.b ** 3 * n_active * 2 * (spec.K // spec.b))
        total_flops = sum(flops.values())
        expert_bytes = spec.K * 2 * spec.n_proj // 2 + 2 * 2 * spec.n_proj * (spec.K // spec.group)
        # the chunked variant materialises each active expert in bf16 (write + read), as the pages do
        chunk_buf_bytes = 0 if args.moe == "fused" else 2 * (2 * spec.K * 2 * spec.n_proj)
        alg_bytes = n_active * (expert_bytes + chunk_buf_bytes) + 2 * spec.T * spec.K + 2 * spec.T * 2 * spec.n_proj
        if args.moe_layer:
            # down projections: GEMM, rotation of h by the down adapter, its Cayley build; the down
            # weights stream through the chunk buffer like gate/up; Y is [T][K]
            nbd = spec.n_proj // spec.b
            flops["gemm_down"] = 2.0 * TK * spec.n_proj * spec.K
            flops["rot_down"] = 2.0 * TK * spec.n_proj * spec.b
            flops["cayley_down"] = 2.0 * spec.b ** 3 * n_active * nbd
            total_flops = sum(flops.values())
            down_bytes = spec.K * spec.n_proj // 2 + 2 * spec.K * (spec.n_proj // spec.group)
            down_buf = 2 * (2 * spec.K * spec.n_proj)
            alg_bytes += n_active * (down_bytes + down_buf) - 2 * spec.T * 2 * spec.n_proj + 2 * spec.T * spec.K
        if backward:
            # dY W^T per routed row, its rotation back, dR, the Cayley backward; the experts stream
            # through the chunk buffer once more; dY and the logits in, dX, dQ and dlogits out
            flops["gemm_bwd"] = gemm_flops
            flops["rot_bwd"] = 2 * 2.0 * TK * spec.K * spec.b * 2
            flops["cayley_bwd"] = 4.0 * spec.b ** 3 * n_active * 2 * (spec.K // spec.b)
            total_flops = sum(flops.values())
            nq = spec.E * 2 * (spec.K // spec.b) * (spec.b * (spec.b - 1) // 2)
            alg_bytes += (n_active * (expert_bytes + chunk_buf_bytes) + 2 * spec.T * 2 * spec.n_proj
                          + 2 * spec.T * spec.K + 2 * spec.T * spec.K + 4 * spec.T * spec.E + 2 * nq + 4 * nq)
    else:
        flops = linear_flops(spec, backward)
        if args.weight_side:
            # the forward rotation on the weight (2 N K b) instead of on the activations (2 M K b P)
            flops["rot_fwd"] = 2.0 * spec.N * spec.K * spec.b
        total_flops = sum(flops.values())
        alg_bytes = weight_bytes(spec) + 2 * spec.M * spec.K + 2 * spec.M * spec.N
        if backward:
            alg_bytes += 2 * spec.M * spec.N + 2 * spec.M * spec.K + 4 * dQ.numel() + 2 * dQ.numel()
    tflops = total_flops / (ms_per_step / 1e3) / 1e12

    # ---- end to end through the public API with host buffers ----
    # Every step copies its own inputs from pinned host memory and reads all of its
    # outputs back into pinned host memory.  Copies in, compute and copies out run on
    # three streams, double-buffered, so step i's read-back and step i+1's upload
    # overlap step i+1's / step i's compute (one step in flight on each engine).
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    host_in = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in inputs.items()}
    for k, v in inputs.items():
        host_in[k].copy_(v)
    dev_in = [{k: torch.empty_like(v) for k, v in inputs.items()} for _ in range(2)]
    dev_out = [new_outputs() for _ in range(2)]
    host_out = [{k: torch.empty(dev_out[b][k].shape, dtype=dev_out[b][k].dtype, pin_memory=True)
                 for k in result_keys} for b in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for b in range(2):  # all buffers free at the start
        ev_comp[b].record(comp)
        ev_out[b].record(comp)

    def e2e_step(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_comp[b])          # compute of step i-2 is done with dev_in[b]
            for k in dev_in[b]:
                dev_in[b][k].copy_(host_in[k], non_blocking=True)
            ev_in[b].record(s_in)
        comp.wait_event(ev_in[b])
        comp.wait_event(ev_out[b])               # read-back of step i-2 is done with dev_out[b]
        d = dev_in[b]
        if is_moe and args.moe_layer:
            step(d["X"], d["logits"], d["Q"], o=dev_out[b], Qdi=d["Q_down"])
        elif is_moe:
            step(d["X"], d["logits"], d["Q"], o=dev_out[b], dYi=d.get("dY"))
        elif backward:
            step(d["X"], d["dY"], d["Q"], o=dev_out[b])
        else:
            step(d["X"], None, d["Q"], o=dev_out[b])
        ev_comp[b].record(comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[b])
            for k in result_keys:
                host_out[b][k].copy_(dev_out[b][k], non_blocking=True)
            ev_out[b].record(s_out)

    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    es, ee = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    es.record(comp)
    s_in.wait_event(es)
    for i in range(args.steps):
        e2e_step(i)
    for b in range(2):
        comp.wait_event(ev_out[b])
    ee.record(comp)
    torch.cuda.synchronize()
    clocks.__exit__(None, None, None)
    clk = clocks.summary()
    e2e_ms = max_over_ranks(es.elapsed_time(ee) / args.steps, dev)
    h2d = sum(v.numel() * v.element_size() for v in host_in.values())
    d2h = sum(v.numel() * v.element_size() for v in host_out[0].values())
    e2e = {"value": tokens * world / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
           "pipelining": "double-buffered: upload, compute and read-back on three streams"}

    # ---- dominant kernel roofline ----
    peak_kind = "copy"
    g_launch = prof.launches["gemm"]
    g_ms = prof.ms["gemm"]
    if is_moe and args.moe == "fused":
        # the grouped fused-dequant GEMM against the tensor peak (no chunk buffer: compute-bound)
        bound = "tensor"
        achieved = flops["gemm"] / (g_ms / args.steps / 1e3) / 1e12
        peak, peak_kind = tensor_peak(peaks, clk)
        unit = "TFLOP/s"
        traffic = None
        kernel = "gemm_dq_kernel, MoE mode (grouped over active experts x gate/up, fused INT4 dequant)"
    elif is_moe:
        # HBM-bound: algorithmic bytes of the whole step ÷ the step (chunk dequant + grouped GEMM dominate)
        bound = "hbm"
        achieved = alg_bytes / (ms_per_step / 1e3) / 1e9
        peak = peaks["hbm_gbs"]
        unit = "GB/s"
        traffic = None
        kernel = ("whole step (chunk dequant + grouped GEMM" + (", forward and backward" if backward else "")
                  + (", gate/up + SwiGLU + down" if args.moe_layer else "") + "), HBM")
    elif spec.M <= 128:
        # few tokens: the weight stream bounds the GEMM; bytes of one launch over its time
        wbytes = weight_bytes(spec)
        per_launch_bytes = wbytes + 2 * spec.P * spec.M * spec.K + 2 * spec.M * spec.N
        avg_s = g_ms / g_launch / 1e3
        bound = "hbm"
        achieved = per_launch_bytes / avg_s / 1e9
        peak = peaks["hbm_gbs"]
        unit = "GB/s"
        traffic = None
        kernel = ("gemm_sm_kernel (small-M split-K fused dequant: TMA-staged codes, 16 decode warps into a "
                  "TMEM operand ring, tcgen05), weight-stream bound at this M" if args.gemm_mode in (0, 5) else
                  "gemm_dq_kernel (fused dequant, tcgen05/TMEM), weight-stream bound at this M")
    else:
        gemm_flops = flops["gemm_fwd"] + flops.get("gemm_bwd", 0.0)
        per_launch = gemm_flops / (g_launch / args.steps)
        avg_s = g_ms / g_launch / 1e3
        bound = "tensor"
        achieved = per_launch / avg_s / 1e12
        peak, peak_kind = tensor_peak(peaks, clk)
        unit = "TFLOP/s"
        # the library's choice: from PLAIN_MIN_TOKENS tokens the bf16 weight copy and the plain
        # GEMM; below, the 2-SM pair kernel for launches of two or more one-CTA waves
        tiles1 = sum(-(-n // 128) for n in spec.splits) * (-(-(-(-spec.M // 192)) // 2))
        if args.gemm_mode == 4:
            kernel = "gemm_bf16_kernel (plain bf16 GEMM, one CTA per tile, tcgen05/TMEM; the weight dequantised first)"
            traffic = gemm_traffic("gemm_bf16_kernel", name)
        elif args.gemm_mode == 3 or (args.gemm_mode == 0 and spec.M >= PLAIN_MIN_TOKENS):
            kernel = ("gemm_bf16_pair_kernel (plain bf16 GEMM on 2-SM pairs, tcgen05 cta_group::2; "
                      "the weight dequantised to bf16 first)")
            traffic = gemm_traffic("gemm_bf16_pair_kernel", name)
        elif args.gemm_mode == 2 or (args.gemm_mode == 0 and tiles1 >= 2 * 148):
            kernel = "gemm_dq2_kernel (fused dequant, 2-SM pair, tcgen05 cta_group::2)"
            traffic = gemm_traffic("gemm_dq2_kernel", name)
        else:
            kernel = "gemm_dq_kernel (fused dequant, tcgen05/TMEM)"
            traffic = None
        if args.weight_side and not backward:
            traffic = None
            kernel = ("gemm_bf16_kernel (plain bf16 x bf16, one CTA per tile; weight-side rotation)" if args.gemm_mode == 4
                      else "gemm_bf16_pair_kernel (plain bf16 x bf16 on 2-SM pairs; weight-side rotation)")
    roofline = {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
                "traffic": traffic, "kernel": kernel,
                "peak_source": f"{peak_src} ({peak_kind})"}

    if rank != 0:
        return None
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        if is_moe:
            cpu = cpu_baseline_moe(case, dY=dY if backward else None, down=dn if args.moe_layer else None)
        else:
            cpu = cpu_baseline_linear(case, backward)
    config = workload_config(name, tokens, world, backward, args, n_active if is_moe else None)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; shapes and distributions of the workload)",
        "config": config, "tflops": tflops, "algorithmic_flops_per_step": total_flops,
        "algorithmic_bytes_per_step": alg_bytes, "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": int(sum(prof.launches.values())),
        "profiled_pass": {"ms_per_step": ms_profiled,
                          "note": "the same K steps again with CUDA events around every library kernel; "
                                  "kernel_ms_per_step and roofline.achieved come from this pass"},
        "kernel_ms_per_step": {k: v / args.steps for k, v in prof.ms.items()},
        "kernel_launches_per_step": {k: v / args.steps for k, v in prof.launches.items()},
        **({"part_ms_per_step": part_ms} if part_ms is not None else {}),
        "clocks": clk,
    }
    return line


# keys of a workload's own line kept in the headline line's "workloads" object
WORKLOAD_KEYS = ("value", "unit", "ms_per_step", "tflops", "config", "algorithmic_flops_per_step",
                 "algorithmic_bytes_per_step", "roofline", "cpu_baseline", "e2e", "gpu_launches", "profiled_pass",
                 "kernel_ms_per_step", "kernel_launches_per_step", "part_ms_per_step", "clocks")


def run_reference(args, rank, world):
    """The oracle (float64 numpy, as it stands) timed on the host cores, on a
    bounded sample of the same workload per step."""
    if rank != 0:
        return None
    from gen import LINEAR_CONFIGS, MOE_CONFIGS, make_linear_case, make_moe_case, make_moe_down, make_moe_grad
    name = args.workload
    n_active = None
    if moe_spec(name) is not None:
        import numpy as np
        import torch
        from oracle import moe_ref
        sys.path.insert(0, os.path.join(ROOT, "tests"))
        from npcase import raw
        spec = moe_spec(name)
        dev = "cuda" if torch.cuda.is_available() else "cpu"
        case = make_moe_case(spec, device=dev)
        dY = make_moe_grad(spec, device=dev) if args.moe_backward else None
        dn = make_moe_down(spec, device=dev) if args.moe_layer else None
        idx, _ = moe_ref.topk(raw(case["logits"]), spec.top_k)
        n_active = int(np.unique(idx).size)
        backward = args.moe_backward
        tokens = full_tokens = spec.T
        per = max(2.0, 150.0 / (args.steps + args.warmup))
        for _ in range(args.warmup):
            cpu_baseline_moe(case, budget_s=per / 4, dY=dY, down=dn)
        res = [cpu_baseline_moe(case, budget_s=per, dY=dY, down=dn) for _ in range(args.steps)]
        value = statistics.mean(r["value"] for r in res)
        sample = res[-1]["sample"]
    else:
        spec = linear_spec(name)
        backward = spec.backward
        tokens = full_tokens = spec.M
        case = make_linear_case(spec)
        per_budget = 150.0 / (args.steps + args.warmup)
        tokens = min(spec.M, 64)
        dt = oracle_linear_step(case, tokens, spec.backward)
        while dt * 2 < per_budget and tokens < spec.M:
            tokens = min(spec.M, tokens * 2)
            dt = oracle_linear_step(case, tokens, spec.backward)
        for _ in range(args.warmup):
            oracle_linear_step(case, tokens, spec.backward)
        times = [oracle_linear_step(case, tokens, spec.backward) for _ in range(args.steps)]
        ms = 1e3 * statistics.mean(times)
        value = tokens / (ms / 1e3)
        sample = f"first {tokens} of {spec.M} tokens per step, float64 numpy ({cpu_model()})"
    ms_per_step = None if moe_spec(name) is not None else ms
    return {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            # the workload's own config (as in our arm's line); the bounded sample each step
            # times is described under cpu_baseline
            "config": workload_config(name, full_tokens, world, backward, args, n_active),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="c4", choices=sorted(WORKLOAD_NAMES),
                    help="the headline workload (default: the MXFP4 training step, the largest that fits one GPU)")
    ap.add_argument("--also", default="c0,c1,c2,c3,c1-m64,c4-m64",
                    help="comma-separated workloads timed after the headline one on a single GPU and reported "
                         "under 'workloads' in the same line ('' for none)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--moe-backward", action="store_true",
                    help="MoE workload: time forward + adapter backward (chunked path)")
    ap.add_argument("--gemm-mode", type=int, default=0, choices=[0, 1, 2, 3, 4],
                    help="GEMM path of the dense workloads (oft_set_gemm_mode): 0 by size (the small-M split-K "
                         "kernel up to 128 tokens), 1 one-CTA fused, 2 2-SM pair fused, 3 bf16 copy + plain pair "
                         "GEMM, 4 bf16 copy + plain one-CTA GEMM")
    ap.add_argument("--weight-side", action="store_true",
                    help="dense workloads: the weight-side rotation variant of the forward")
    ap.add_argument("--moe-layer", action="store_true",
                    help="MoE workload: time the full expert layer (gate/up, SwiGLU, down projection)")
    ap.add_argument("--moe", default="chunked", choices=["chunked", "fused"],
                    help="MoE workload: the pages' chunked dequant (default) or the fused-dequant grouped GEMM")
    args = ap.parse_args(argv)
    if args.moe_layer and args.moe_backward:
        ap.error("--moe-layer times the forward of the full expert layer; --moe-backward the gate/up backward")
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU: start the ranks and hand back their exit status
        import subprocess
        import socket
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        argv = sys.argv[1:] if argv is None else list(argv)
        sys.exit(subprocess.call(launch_cmd(argv, args.gpus, port)))
    if args.impl == "reference":
        rank, world, _ = dist_env()
        line = run_reference(args, rank, world)
    else:
        rank, world = init_dist("nccl")
        if world != args.gpus:
            print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
        line = run_ours(args, rank, world, args.workload)
        # the other workloads, on a single GPU only (no collective runs in this loop)
        extras = [w for w in args.also.split(",") if w and w != args.workload] if world == 1 else []
        if extras and line is not None:
            line["workloads"] = {}
            for name in extras:
                import gc
                import torch
                gc.collect()
                torch.cuda.empty_cache()
                try:
                    sub = run_ours(args, rank, world, name)
                    line["workloads"][name] = {k: sub[k] for k in WORKLOAD_KEYS if k in sub}
                except Exception as exc:  # reported, never fatal to the headline line
                    line["workloads"][name] = {"error": repr(exc)[:300]}
        import torch.distributed as dist
        if dist.is_initialized():
            dist.barrier()
            dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
