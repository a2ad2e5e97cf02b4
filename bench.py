"""Benchmark of the KATA chunked-state causal forward (one JSON line).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one kata_fwd_chunked call over one batch of the long-context
workload (B=1, H=16, T=131072, d_k=32, d_v=64, C=128, bf16 inputs, fp32
accumulation; PSD feature), inputs resident in HBM. With N > 1 (launched by
torch.distributed.run) every rank runs its own batch (weak scaling, no
collective on the data path); the step time is the max over ranks.

The per-step input (805 MB) is larger than the 126 MB L2, so no L2 flush is
needed between steps.
"""

from __future__ import annotations

import argparse
import hashlib
from dataclasses import replace
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

W_DECODE_BATCH = 256
METRIC = "KATA causal fwd tokens/sec at T=131072 (chunked) and % of tensor/HBM roofline"
UNIT = "tokens/s"
NOMINAL_FP32_TFLOPS_PER_SM_GHZ = 128 * 2 / 1000.0   # 128 FP32 lanes x FMA, per GHz, in TFLOP/s

# Which roofline each of the library's kernels is held to.
#   tensor: bf16 tensor-core contraction;  alu: fp32 FFMA on the CUDA cores;
#   hbm: streaming kernel.
KERNEL_BOUND = {
    "tc_quadratic": "tensor",
    "tc_fo_pass": "hbm",
    "tc_fo_increment": "hbm",
    "simt_segment_pass": "alu",
    "simt_segment_increment": "alu",
    "simt_quadratic": "alu",
    "simt_decode": "hbm",
    "simt_bwd_dq": "alu",
    "simt_bwd_dkdv": "alu",
    "simt_bwd_prefix_increment": "alu",
    "simt_bwd_suffix_increment": "alu",
    "simt_delta": "alu",
}
METRIC_BWD = "KATA causal bwd (dq, dk, dv) tokens/sec at T=131072 (chunked)"


def state_rows(d_k, feature):
    """D, the state rows of a feature (PSD, first-order, KATA-Mg / Sigma-g
    with g = 2 over the two halves of the key)."""
    h = d_k // 2
    return {"psd": d_k * (d_k + 1) // 2, "first_order": d_k + 1, "mg2": h * (h + 1),
            "sigma_g2": h * (h + 1) // 2}[feature]


def pair_weight_flops(d_k, feature):
    """Flops of one query-key weight in closed form: the dot product(s) and
    their squares (PSD (q.k)^2; first-order 1 + q.k; Mg2 two half-dots;
    Sigma-g2 four half-dots)."""
    return {"psd": 2 * d_k + 1, "first_order": 2 * d_k + 1, "mg2": 2 * d_k + 3,
            "sigma_g2": 4 * d_k + 7}[feature]


def algorithmic_per_token_head(d_k, d_v, C, feature="psd"):
    """(flops, bytes) the chunked forward must do per token-head: the causal
    half of the intra-chunk block (each pair: its weight, the d_v
    multiply-adds of the value and the normaliser's add), the state update
    and the readout; bf16 q, k, v read once and o written once."""
    D = state_rows(d_k, feature)
    intra = (C + 1) / 2 * (pair_weight_flops(d_k, feature) + 2 * d_v + 1)
    update = 2 * D * d_v + D
    readout = 2 * D * d_v + 2 * D
    return intra + update + readout, (2 * d_k + d_v) * 2 + d_v * 2


def algorithmic_delta_per_token_head(d_k, d_v):
    """(flops, bytes) of the DeltaKATA rule per token-head, as the recurrence
    states it: the stored binding phi~(k)^T S', the rank-one write and the
    readout phi~(q)^T S', each over the D x (d_v + 1) augmented state; bf16
    q, k, v and fp32 beta read once, o written once."""
    D = state_rows(d_k, "psd")
    return 6 * D * (d_v + 1), (2 * d_k + d_v) * 2 + 4 + d_v * 2


def feature_products_per_token_head(d_k, feature="psd"):
    """Scalar products the feature expansion needs per token-head: phi(k) for
    the state update and phi~(q) for the readout, one product per packed
    feature each (the query's multiplicity 2 folds into its product; a
    Sigma-g2 feature sums two). The first-order feature [1, u] is the input
    itself and needs none."""
    if feature == "first_order":
        return 0
    per = 2 if feature == "sigma_g2" else 1
    return 2 * per * state_rows(d_k, feature)


def algorithmic_backward_per_token_head(d_k, d_v, C, feature="psd"):
    """(flops, bytes) the gradient of the chunked forward must do per
    token-head: the carried parts of dq (S g + z c, then the query feature's
    Jacobian), dk (R v + r, the key feature's Jacobian) and dv (R^T phi(k)),
    the updates of the prefix and suffix states, the normaliser and g, c; the
    causal half of the intra-chunk pairs (q.k, g.v, dq, dk, dv, w); bf16 q, k,
    v, dout read once and dq, dk, dv written once. The kernels also recompute
    dout . y from the numerator; that recomputation is not counted."""
    D = d_k * (d_k + 1) // 2 if feature == "psd" else d_k + 1
    carried = (2 * D * d_v + 6 * D) + (2 * D * d_v + 6 * D) + (2 * D * d_v + D)
    updates = (2 * D * d_v + 2 * D) + (2 * D * d_v + 3 * D)
    norm = 2 * D + 3 * d_v
    intra = (C + 1) / 2 * (6 * d_k + 4 * d_v + 4)
    return carried + updates + norm + intra, (4 * d_k + 3 * d_v) * 2


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                "sm_max_mhz": p.get("sm_max_mhz", 1965.0), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "sm_max_mhz": 1965.0, "source": "fallback"}


# Source files that define each profiled kernel (a recorded traffic figure is
# valid only while these are unchanged).
KERNEL_SOURCES = {
    "tc_segment_pass": ["chunked_tc.cu", "psd_tc_common.cuh", "tc_common.cuh", "common.cuh"],
    "tc_segment_increment": ["chunked_tc.cu", "psd_tc_common.cuh", "tc_common.cuh", "common.cuh"],
    "tc_quadratic": ["quadratic_tc.cu", "tc_common.cuh", "common.cuh"],
    "tc_fo_pass": ["fo_tc.cu", "tc_common.cuh", "common.cuh"],
    "tc_fo_increment": ["fo_tc.cu", "tc_common.cuh", "common.cuh"],
    "tc_bwd_dq": ["bwd_tc.cu", "psd_tc_common.cuh", "tc_common.cuh", "common.cuh"],
    "tc_bwd_dkdv": ["bwd_tc.cu", "psd_tc_common.cuh", "tc_common.cuh", "common.cuh"],
    "tc_bwd_suffix_increment": ["chunked_tc.cu", "psd_tc_common.cuh", "tc_common.cuh", "common.cuh"],
    "tc_variant_pass": ["var_tc.cu", "psd_tc_common.cuh", "tc_common.cuh", "common.cuh"],
    "tc_variant_increment": ["var_tc.cu", "psd_tc_common.cuh", "tc_common.cuh", "common.cuh"],
}


def source_hash(kernel=None):
    """Hash of the kernel's source files (all of csrc when the kernel has no
    entry in KERNEL_SOURCES)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "kernelized_linear_attention_kata_b200", "csrc")
    names = KERNEL_SOURCES.get(kernel) or sorted(
        fn for fn in os.listdir(csrc) if fn.endswith((".cu", ".cuh", ".h")))
    for fn in sorted(names):
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current sources of that kernel; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(kernel)
    if not rec or rec.get("source_sha") != source_hash(kernel):
        return None
    return rec.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples taken during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        rows = []
        for l in getattr(self, "lines", []):
            parts = [p.strip() for p in l.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append({"sm": float(parts[1]), "max": float(parts[2]), "power": float(parts[3]),
                             "hw": parts[5], "hw_thermal": parts[6], "sw_thermal": parts[7],
                             "sw_power": parts[8]})
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        loaded = [r for r in rows if r["power"] > 200.0] or rows
        reasons = set()
        for r in loaded:
            for key, name in (("hw", "hw_slowdown"), ("hw_thermal", "hw_thermal_slowdown"),
                              ("sw_thermal", "sw_thermal_slowdown"), ("sw_power", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded),
                "sm_max_mhz": max(r["max"] for r in rows), "reasons": sorted(reasons),
                "samples": len(loaded)}


# ---------------------------------------------------------------------------
# CPU oracle (baseline leg and --impl reference arm)
# ---------------------------------------------------------------------------

def host_cores():
    """CPU cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


_THREAD_ENV = ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")


def _oracle_head(job):
    """One worker's share of the CPU baseline: the oracle's chunked forward on
    the first `n` tokens of head (b, h), read from the inputs' .npy files.
    Returns the seconds it took."""
    import numpy as np

    import oracle as O
    folder, b, h, n, C, feature = job
    q, k, v = (np.asarray(np.load(os.path.join(folder, f"{x}.npy"), mmap_mode="r")[b, h, :n],
                          dtype=np.float64) for x in "qkv")
    t0 = time.perf_counter()
    O.forward_chunked(q, k, v, C, feature)
    return time.perf_counter() - t0


class OracleBaseline:
    """The fp64 oracle timed on the host's cores: one process per head (spawned,
    one BLAS thread each), each running the oracle's chunked forward on its
    head. A round runs min(cores, B*H) heads at once on the first `n` tokens
    of each (the causal forward of a prefix is the prefix of the forward), `n`
    chosen so that a round takes about the budget; the rate is tokens of the
    workload (token-heads / H) per second of wall time."""

    def __init__(self, w):
        import tempfile

        import numpy as np

        from kernelized_linear_attention_kata_b200 import workloads as W
        self.w = w
        self.cores = min(host_cores(), w.B * w.H)
        base = "/dev/shm" if os.path.isdir("/dev/shm") else None
        self.folder = tempfile.mkdtemp(prefix="kata_oracle_", dir=base)
        for name, t in zip("qkv", W.make_inputs(w)):
            # the bf16-rounded inputs, exactly, as float32
            np.save(os.path.join(self.folder, f"{name}.npy"), t.float().numpy())
        import multiprocessing as mp
        saved = {k: os.environ.get(k) for k in _THREAD_ENV}
        for k in _THREAD_ENV:
            os.environ[k] = "1"
        try:
            # spawn, not fork: the parent may already hold a CUDA context
            self.pool = mp.get_context("spawn").Pool(self.cores)
        finally:
            for k, val in saved.items():
                if val is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = val
        self.n = min(w.T, 4 * w.C)
        self.rate_per_token = None

    def round(self, budget_s):
        """One timed round. Returns (tokens/s, seconds, description)."""
        w = self.w
        if self.rate_per_token is not None:
            n = int(budget_s / self.rate_per_token) // w.C * w.C
            self.n = max(w.C, min(w.T, n))
        heads = [divmod(bh, w.H) for bh in range(w.B * w.H)][:self.cores]
        jobs = [(self.folder, b, h, self.n, w.C, w.feature) for b, h in heads]
        t0 = time.perf_counter()
        per_head = self.pool.map(_oracle_head, jobs, chunksize=1)
        dt = time.perf_counter() - t0
        self.rate_per_token = max(per_head) / self.n
        token_heads = len(heads) * self.n
        desc = (f"oracle forward_chunked (fp64 numpy, one process and one BLAS thread per head) on "
                f"{len(heads)} of {w.B * w.H} heads at once, first {self.n} of {w.T} tokens each, "
                f"of {w.name}: {dt:.2f} s; tokens/s = token-heads / H / s")
        return token_heads / w.H / dt, dt, desc

    def close(self):
        import shutil
        self.pool.terminate()
        self.pool.join()
        shutil.rmtree(self.folder, ignore_errors=True)


def oracle_sample(w, budget_s):
    """The CPU baseline beside the GPU number: a calibration round, then one
    round of about `budget_s` seconds. Returns (tokens/s, cores, description)."""
    base = OracleBaseline(w)
    try:
        base.round(budget_s / 10)
        value, _, desc = base.round(budget_s)
        return value, base.cores, desc
    finally:
        base.close()


def run_reference(args, rank, world):
    from kernelized_linear_attention_kata_b200 import workloads as W
    if rank != 0:
        return 0
    w = W.WORKLOADS[args.workload]
    budget = args.ref_step_budget or max(0.5, 150.0 / (args.steps + args.warmup))
    base = OracleBaseline(w)
    try:
        base.round(budget / 10)                      # calibration of the sample size
        for _ in range(args.warmup):
            base.round(budget)
        vals, secs = [], []
        sample = ""
        for _ in range(args.steps):
            v, dt, sample = base.round(budget)
            vals.append(v)
            secs.append(dt)
    finally:
        base.close()
    value = statistics.mean(vals)
    ms_per_step = 1000.0 * statistics.mean(secs)
    full_step_ms = 1000.0 * w.B * w.T / value
    sample += (f"; a step is one such round ({ms_per_step:.0f} ms); the whole workload "
               f"(B x T tokens) at this rate would take {full_step_ms:.0f} ms")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": base.cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "projected_full_step_ms": full_step_ms,
    }
    print(json.dumps(line), flush=True)
    return 0


def max_over_ranks(x, world, device):
    """The largest x of all ranks (every rank gets it): a multi-GPU time is
    the slowest rank's."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(ms_per_step, tokens_per_step, world, device):
    """Whole-job tokens/s of `world` replicas, each processing tokens_per_step
    per step: all ranks' tokens over the slowest rank's step time."""
    ms = max_over_ranks(ms_per_step, world, device)
    return world * tokens_per_step / (ms / 1e3), ms


def workload_config(w, world=1):
    return {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "d_k": w.d_k, "d_v": w.d_v,
            "C": w.C, "feature": w.feature, "form": "chunked (segmented scan carry)",
            "l2": "inputs larger than L2 (no flush needed)", "parallelism": f"replicas x{world}"}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from kernelized_linear_attention_kata_b200 import api
    from kernelized_linear_attention_kata_b200 import build as kbuild
    from kernelized_linear_attention_kata_b200 import workloads as W

    torch.cuda.set_device(local_rank)
    kbuild.build()
    dev = torch.device("cuda", local_rank)
    form = args.form
    fo = form in ("first_order", "first_order_sequential")
    w = W.WORKLOADS[args.workload if not fo else "first_order64k_bf16"]
    if args.feature:
        if fo or form in ("backward", "delta"):
            raise SystemExit("--feature applies to the chunked, sequential, quadratic forms")
        w = replace(w, feature=args.feature)
    if form == "quadratic":
        w = w.with_T(args.T or W.LONG_QUADRATIC_T)
    elif args.T:
        w = w.with_T(args.T)
    seq = args.shard == "sequence"
    if seq and (form != "chunked" or w.T % world):
        raise SystemExit("--shard sequence needs --form chunked and T divisible by the ranks")
    if not seq:
        w = replace(w, seed=w.seed + 1000 * rank)     # one seeded batch per rank
    stream = torch.cuda.current_stream()
    phi_th = 0            # feature-expansion products per token-head, where the form has them
    if form == "decode":
        B, H = args.decode_batch, W.DECODE_HEADS
        q, k, v = W.make_decode_inputs(B, H, device=dev)
        # prior state per sequence: 4096 seeded tokens accumulated by the library
        kp, vp = W.make_decode_prior_tokens(B, H, device=dev)
        _, S, z = api.fwd_chunked(kp, kp, vp, 128, "psd", return_state=True)
        del kp, vp
        o = torch.empty_like(v)
        ws = None

        def step():
            api.kata_decode_step(q, k, v, S, z, o)
        tokens_per_step = B
        token_heads = B * H
        D = api.state_dim(W.DECODE_DK)
        flops_th = 2 * D * W.DECODE_DV * 2 + 3 * D
        bytes_th = 2 * 4 * D * (W.DECODE_DV + 1) + 2 * (2 * W.DECODE_DK + 2 * W.DECODE_DV)
        phi_th = feature_products_per_token_head(W.DECODE_DK)
        config = {"workload": f"decode_b{B}_h{H}", "B": B, "H": H, "d_k": W.DECODE_DK,
                  "d_v": W.DECODE_DV, "feature": "psd", "form": "decode step",
                  "l2": "state larger than L2 (no flush needed)"}
    else:
        q, k, v = W.make_inputs(w, device=dev)
        o = torch.empty_like(v)
        if form == "backward":
            dy = W.make_grad_output(w, device=dev)            # seeded dL/dy
            dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
            nb = api.bwd_chunked_workspace_bytes(w.B, w.H, w.T, w.d_k, w.d_v, w.C, q.dtype, w.feature)
            ws = torch.empty(nb, dtype=torch.uint8, device=dev)

            def run_on(ins, outs):
                api.kata_bwd_chunked(*ins, *outs, w.C, w.feature, workspace=ws)
            flops_th, bytes_th = algorithmic_backward_per_token_head(w.d_k, w.d_v, w.C, w.feature)
            e2e_in, e2e_out = [q, k, v, dy], [dq, dk, dv]
        elif form == "delta":
            beta = W.make_delta_beta(w.B, w.H, w.T, w.seed, device=dev)
            ws = torch.empty(256, dtype=torch.uint8, device=dev)

            def run_on(ins, outs):
                api.kata_fwd_delta(*ins, beta, *outs, w.feature, workspace=ws)
            flops_th, bytes_th = algorithmic_delta_per_token_head(w.d_k, w.d_v)
            phi_th = 3 * state_rows(w.d_k, "psd")
        elif form == "quadratic":
            ws = None

            def run_on(ins, outs):
                api.kata_fwd_quadratic(*ins, *outs, w.feature)
            flops_th = (w.T + 1) / 2 * (2 * w.d_k + 2 * w.d_v + 2)
            _, bytes_th = algorithmic_per_token_head(w.d_k, w.d_v, w.C, w.feature)
        elif seq:
            # one sequence cut along T, this rank's slice of it
            from kernelized_linear_attention_kata_b200 import sequence_parallel as SP
            Tr = w.T // world
            sl = (slice(None), slice(None), slice(rank * Tr, (rank + 1) * Tr))
            q, k, v = (t[sl].contiguous() for t in (q, k, v))
            o = torch.empty_like(v)
            w = w.with_T(Tr)
            ws = None

            def run_on(ins, outs):
                SP.fwd_chunked_sequence_parallel(*ins, w.C, w.feature, out=outs[0])
            flops_th, bytes_th = algorithmic_per_token_head(w.d_k, w.d_v, w.C, w.feature)
            phi_th = feature_products_per_token_head(w.d_k, w.feature)
        else:
            ws = api.alloc_workspace(w.B, w.H, w.T, w.d_k, w.d_v, w.C, q.dtype, w.feature, dev)
            seq_carry = form in ("sequential", "first_order_sequential")

            def run_on(ins, outs):
                api.kata_fwd_chunked(*ins, *outs, w.C, w.feature, workspace=ws, sequential=seq_carry)
            flops_th, bytes_th = algorithmic_per_token_head(w.d_k, w.d_v, w.C, w.feature)
            phi_th = feature_products_per_token_head(w.d_k, w.feature)
        if form != "backward":
            e2e_in, e2e_out = [q, k, v], [o]

        def step():
            run_on(e2e_in, e2e_out)
        tokens_per_step = w.B * w.T
        token_heads = w.B * w.H * w.T
        config = workload_config(w)
        config["form"] = {"chunked": "chunked (segmented scan carry)",
                          "sequential": "chunked (sequential carry)",
                          "first_order": "chunked first-order (segmented scan carry)",
                          "first_order_sequential": "chunked first-order (sequential carry)",
                          "quadratic": "quadratic (flash-style)",
                          "delta": "DeltaKATA (delta-rule state, chunked triangular solve)",
                          "backward": "gradient of the chunked form (prefix and suffix scans)"}[form]

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if ws is not None:
        st = api.kata_workspace_status(ws)
        if st != 0:
            raise RuntimeError(f"device status {st} after warm-up")

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clocks:
        api.profile_enable(True)
        barrier()
        torch.cuda.synchronize()
        start.record(stream)
        for _ in range(args.steps):
            step()
        end.record(stream)
        torch.cuda.synchronize()
        barrier()
        prof = api.profile_read()
        api.profile_enable(False)
    ms = start.elapsed_time(end) / args.steps
    value, ms = aggregate_throughput(ms, tokens_per_step, world, dev)

    # roofline of the dominant kernel, timed live by the library's events
    peaks = load_peaks()
    dom = max(prof, key=lambda n: prof[n][1])
    launches, dom_ms = prof[dom]
    dom_avg_s = dom_ms / launches / 1e3
    # achieved = the step's algorithmic work / one launch of the dominant kernel
    per_launch_units = token_heads
    bound = KERNEL_BOUND.get(dom, "tensor")
    timed_s = ms * args.steps / 1e3
    if bound == "hbm":
        achieved = bytes_th * per_launch_units / dom_avg_s / 1e9
        peak, unit, peak_kind = peaks["hbm_gbs"], "GB/s", peaks["source"]
    elif bound == "alu":
        achieved = flops_th * per_launch_units / dom_avg_s / 1e12
        peak = 148 * NOMINAL_FP32_TFLOPS_PER_SM_GHZ * peaks["sm_max_mhz"] / 1000.0
        unit, peak_kind = "TFLOP/s", "derived: 148 SMs x 128 FP32 FMA lanes x 2 x max SM clock"
    else:
        achieved = flops_th * per_launch_units / dom_avg_s / 1e12
        sustained = timed_s > 1.0
        peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
        unit = "TFLOP/s"
        peak_kind = f"{peaks['source']} bf16 {'sustained' if sustained else 'burst'}"
    scope = "dominant kernel (it carries the step's whole algorithmic work)"
    if form == "backward":
        # the work is split over four kernels: hold the whole step to the roofline
        achieved = flops_th * per_launch_units / (ms / 1e3) / 1e12
        scope = "whole step (four kernels share the work)"
    roofline = {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                "frac": achieved / peak, "traffic": recorded_traffic(dom), "kernel": dom,
                "kernel_ms": dom_ms / launches, "peak_kind": peak_kind, "scope": scope,
                "step_frac_of_tensor_or_hbm": None}
    # whole-step fraction of the binding tensor/HBM roofline of the method
    t_tensor = flops_th * token_heads / (peaks["bf16_tflops"] * 1e12)
    t_hbm = bytes_th * token_heads / (peaks["hbm_gbs"] * 1e9)
    roofline["step_frac_of_tensor_or_hbm"] = max(t_tensor, t_hbm) / (ms / 1e3)
    # third floor: the feature expansion's products on the FP32 lanes
    if phi_th:
        lanes_per_s = 148 * 128 * peaks["sm_max_mhz"] * 1e6
        floor_s = phi_th * token_heads / lanes_per_s
        roofline["phi_alu"] = {"products_per_token_head": phi_th, "floor_ms": floor_s * 1e3,
                               "frac_of_step": floor_s / (ms / 1e3),
                               "peak_kind": "derived: 148 SMs x 128 FP32 lanes x max SM clock"}
    gpu_launches = sum(n for n, _ in prof.values())

    # end to end through the public API with pinned host buffers
    e2e = None
    if not args.no_e2e and form != "decode":
        hosts_in = [t.cpu().pin_memory() for t in e2e_in]
        hosts_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in e2e_out]

        # A serving loop: step i's inputs go in on one copy stream, its result
        # comes back on another, and the device buffers alternate between two
        # sets, so that step i + 1's inputs cross the link while step i
        # computes and step i - 1's result leaves. Each step's compute waits
        # for its own inputs and for the result last computed in its buffer
        # set (two steps back) to have left; each copy in waits for the
        # compute that last read its buffer set.
        ins_sets = [e2e_in, [torch.empty_like(t) for t in e2e_in]]
        outs_sets = [e2e_out, [torch.empty_like(t) for t in e2e_out]]
        h2d_s, d2h_s = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        last = [{"compute": None, "out": None}, {"compute": None, "out": None}]
        count = [0]

        def e2e_step():
            b = count[0] % 2
            count[0] += 1
            ins, outs = ins_sets[b], outs_sets[b]
            ev_in, ev_comp, ev_out = (torch.cuda.Event() for _ in range(3))
            with torch.cuda.stream(h2d_s):
                if last[b]["compute"] is not None:
                    h2d_s.wait_event(last[b]["compute"])       # this set's inputs no longer read
                for d, h in zip(ins, hosts_in):
                    d.copy_(h, non_blocking=True)
                ev_in.record(h2d_s)
            stream.wait_event(ev_in)
            if last[b]["out"] is not None:
                stream.wait_event(last[b]["out"])              # this set's outputs copied out
            run_on(ins, outs)
            ev_comp.record(stream)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(ev_comp)
                for h, d in zip(hosts_out, outs):
                    h.copy_(d, non_blocking=True)
                ev_out.record(d2h_s)
            last[b] = {"compute": ev_comp, "out": ev_out}

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        barrier()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(2, args.steps)                    # the same K steps as the device timing
        s2.record(h2d_s)
        for _ in range(n_e2e):
            e2e_step()
        e2.record(d2h_s)
        torch.cuda.synchronize()
        ms_e2e = s2.elapsed_time(e2) / n_e2e
        e2e_value, ms_e2e = aggregate_throughput(ms_e2e, tokens_per_step, world, dev)
        e2e = {"value": e2e_value, "unit": UNIT,
               "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in e2e_in),
               "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in e2e_out),
               "ms_per_step": ms_e2e,
               "overlap": "two device buffer sets: step i+1 in, step i computing and step i-1 "
                          "out at once, on two copy streams and the compute stream"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and form == "chunked":
        val, cores, sample = oracle_sample(W.WORKLOADS[args.workload], budget_s=args.cpu_budget)
        cpu = {"value": val, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}

    if rank == 0:
        line = {
            "metric": METRIC_BWD if form == "backward" else METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "strong" if seq else "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config | {"parallelism": f"sequence x{world}" if seq else f"replicas x{world}"},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": gpu_launches,
            "kernels": {n: {"launches": c, "avg_ms": t / c} for n, (c, t) in prof.items()},
            "clocks": clocks.summary(), "token_heads_per_s": value * token_heads / tokens_per_step,
        }
        print(json.dumps(line), flush=True)
    return 0


def launch_ranks(n):
    """Re-run this command as n local ranks under torch.distributed.run
    (127.0.0.1 rendezvous on a free port); rank 0 prints the JSON line. The
    exit status is the launcher's."""
    import socket
    with socket.socket() as sock:
        sock.bind(("127.0.0.1", 0))
        port = sock.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__),
           *sys.argv[1:]]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=None,
                    help="GPUs (ranks) on this node; without a torch.distributed launcher in "
                         "the environment, bench.py starts that many ranks itself")
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="long131k_bf16")
    ap.add_argument("--form", default="chunked",
                    choices=["chunked", "sequential", "first_order", "first_order_sequential",
                             "quadratic", "decode", "backward", "delta"],
                    help="chunked is the headline; the others are secondary measurements")
    ap.add_argument("--shard", choices=["heads", "sequence"], default="heads",
                    help="heads: independent replicas, one batch per rank (weak scaling); "
                         "sequence: one sequence cut along T, one slice per rank, one all-reduce "
                         "of the slice states (strong scaling)")
    ap.add_argument("--feature", choices=["psd", "mg2", "sigma_g2"], default=None,
                    help="feature map of the chunked / sequential / quadratic forms (default: the "
                         "workload's, PSD); mg2 and sigma_g2 are KATA-Mg and KATA-Sigma-g, g = 2")
    ap.add_argument("--decode-batch", type=int, default=W_DECODE_BATCH)
    ap.add_argument("--T", type=int, default=0, help="override T (profiling a smaller case)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work")
    ap.add_argument("--ref-step-budget", type=float, default=0.0,
                    help="seconds of oracle work per reference step (default: 150 s / (K + W))")
    args = ap.parse_args()

    if "WORLD_SIZE" not in os.environ and (args.gpus or 1) > 1:
        return launch_ranks(args.gpus)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus is not None and args.gpus != world:
        raise SystemExit(f"--gpus {args.gpus} but the launcher started {world} ranks")
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        return run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
