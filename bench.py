#!/usr/bin/env python3
"""Throughput of libsa3 (microscaled-FP4 attention forward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl sa3|reference]

One step = the whole hot path on one batch: sa3_quantize_qkv (K smoothing
+ FP4 microscaling of Q, K, V) followed by sa3_attn_fwd, on the non-causal
workload B=2, H=16, N=4096, d=128 (seeded synthetic bf16 inputs already
resident in HBM).  The metric is attention TOPS = 4*B*H*N^2*d / t.
L2 is flushed before every timed step (a 256 MiB write, then a 256 MiB read
of another buffer, so that no input is cached and the timed kernels do not
pay for writing back the flush's dirty lines); each step is timed
with CUDA events on the launching stream, with a barrier and a device
synchronize around the K timed steps; multi-GPU runs take the maximum
over ranks and report the whole-job rate (every rank runs its own batch:
weak scaling, no data-path collective).

Options: --variant i8 times the 8-bit variant (INT8 QK^T, FP16 P V) and
i8_train its training forward (also writes the per-row log-sum-exp);
--workload picks another seeded workload; --nq gives Q fewer or more tokens
than K and V (ops then count the (query, key) pairs the mask leaves);
--p-two-level times the two-level P recipe.

--impl reference runs the CPU oracle (oracle/) as it stands on the host
cores, on a bounded sample of the same workload, and prints the same line
with "impl": "reference".
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import sa3_inputs  # noqa: E402

WORKLOAD = "noncausal_b2h16n4096d128"
METRIC = "attention TOPS (4*B*H*N^2*d/t) and % of B200 dense FP4 peak, 1 GPU"
UNIT = "TOPS"
FP4_DATASHEET_TOPS = 9000.0        # NVIDIA B200 dense FP4 (18 PF with 2:4 sparsity)
FP4_PER_BF16 = 4.0                 # nominal dense FP4 / bf16 ratio (9 / 2.25 PF)
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20
LAUNCHES_PER_STEP = 3              # sa3_quantize_qkv: 2 kernels; sa3_attn_fwd: 1
EX2_PER_SM_CLK = 16                # ex2.approx.ftz.f32 results per SM per clock (measured on a B200)
EX2_PER_S = 1.0 + 1.0 / 16 + 1.0 / 64  # FP4 attention: P, one block scale per 16 keys, alpha per row half


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="sa3", choices=["sa3", "reference"])
    ap.add_argument("--workload", default=WORKLOAD, choices=list(sa3_inputs.WORKLOADS))
    ap.add_argument("--variant", default="fp4", choices=["fp4", "i8", "i8_train"],
                    help="fp4: the microscaled FP4 path (the headline); i8: the 8-bit variant "
                         "(INT8 QK^T, FP16 P V); i8_train: the 8-bit forward used for training "
                         "(also writes the per-row log-sum-exp)")
    ap.add_argument("--nq", type=int, default=0,
                    help="query tokens (default: the workload's N); keys and values keep N "
                         "(sa3_*_lens; causal aligns the last query with the last key)")
    ap.add_argument("--p-two-level", action="store_true",
                    help="fp4 only: P pre-scaled by 2^11 before it is microscaled (SA3_P_TWO_LEVEL)")
    ap.add_argument("--v-smooth", action="store_true",
                    help="fp4 only: V smoothed like K, its mean added back after O / l (SA3_V_SMOOTH)")
    ap.add_argument("--q-on-load", action="store_true",
                    help="fp4 only: the quantizer skips Q and the attention kernel quantizes the bf16 Q "
                         "itself (SA3_SKIP_Q + SA3_Q_ON_LOAD); same output bits")
    ap.add_argument("--skip-cpu-baseline", action="store_true",
                    help="omit the oracle timing (for profiler runs)")
    args = ap.parse_args()
    if (args.p_two_level or args.v_smooth or args.q_on_load) and args.variant != "fp4":
        ap.error("--p-two-level, --v-smooth and --q-on-load apply to the fp4 variant only")
    if args.nq < 0:
        ap.error("--nq must be positive")
    return args


def dist_init(n):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n:
        raise SystemExit(f"--gpus {n} but WORLD_SIZE={world}")
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl" if torch.cuda.is_available() else "gloo",
                                             timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return {"bf16_tflops": FALLBACK_BF16_TFLOPS, "bf16_tflops_sustained": 1400.0,
                "hbm_gbs": FALLBACK_HBM_GBS, "sm_max_mhz": 1965.0}, "fallback"


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled every 2 ms through
    NVML while the timed region runs (nvidia-smi's own sampling period is
    too long for a region of a few milliseconds)."""
    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, device: int):
        self.device = device
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self.error = None
        self._stop = threading.Event()

    def _handle(self):
        import pynvml
        pynvml.nvmlInit()
        pr = torch.cuda.get_device_properties(self.device)
        bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
        try:
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.device)

    def __enter__(self):
        try:
            self.nv, self.h = self._handle()
            self.max_mhz = float(self.nv.nvmlDeviceGetMaxClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        except Exception as e:  # pragma: no cover
            self.error = repr(e)
        return self

    def _run(self):
        get_r = getattr(self.nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            self.nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(float(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)))
                r = int(get_r(self.h))
                for n, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(n)
            except Exception as e:  # pragma: no cover
                self.error = repr(e)
                return
            time.sleep(0.002)

    def __exit__(self, *a):
        self._stop.set()
        if hasattr(self, "t"):
            self.t.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"],
                    "samples": 0, "error": self.error}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml, 2 ms"}


def profiled_traffic(kernel_src: str, profile: str):
    """DRAM bytes per launch recorded in a committed ncu summary, or None if
    the kernel source has changed since (sha256 prefix recorded there)."""
    import hashlib
    try:
        src = open(os.path.join(ROOT, kernel_src), "rb").read()
        txt = open(os.path.join(ROOT, "profiles", profile)).read()
    except OSError:
        return None
    sha = hashlib.sha256(src).hexdigest()[:16]
    rec = dict(line.split(": ", 1) for line in txt.splitlines() if line.startswith(("source_sha256_16: ",)))
    if rec.get("source_sha256_16", "").strip() != sha:
        return None
    for line in txt.splitlines():
        if line.startswith("| dram_bytes_per_launch |"):
            return int(line.split("|")[2].strip())
    return None


def fp4_peak_probe(sa3, dev, iters=16384):
    """Block-scaled FP4 tensor-core rate on this GPU (sa3_probe_fp4_mma: one
    CTA per SM, M=128, K=64, N=128 and N=256), timed with CUDA events on the
    launching stream; best of 3 per shape.  Every run's accumulators are
    checked to hold 64*iters (the tensor core did every MMA)."""
    ctas = torch.cuda.get_device_properties(dev).multi_processor_count
    res = {}
    for n in (128, 256):
        sa3.probe_fp4_mma(n=n, iters=256, device=dev)  # warm-up
        best = None
        for _ in range(3):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            out = sa3.probe_fp4_mma(n=n, iters=iters, device=dev)
            e1.record()
            torch.cuda.synchronize(dev)
            if not torch.all(out == 64.0 * iters):
                raise RuntimeError(f"FP4 MMA probe (N={n}) accumulated the wrong values")
            ms = e0.elapsed_time(e1)
            best = ms if best is None else min(best, ms)
        res[f"n{n}_tops"] = round(2.0 * 128 * n * 64 * iters * ctas / (best * 1e-3) / 1e12, 1)
    res["tops"] = max(res["n128_tops"], res["n256_tops"])
    res["how"] = (f"sa3_probe_fp4_mma: {ctas} CTAs x {iters} tcgen05.mma.kind::mxf4nvf4.block_scale "
                  f"(M=128, K=64), best of 3 per N, CUDA events")
    return res


def accuracy_sample(w, q, k, v, out, causal, two=False, vsm=False, nunits=6):
    """The output's accuracy on a seeded sample of (head, Q block) units: the
    oracle quantizes those heads itself and attends on its own operands
    (worst per-block rel-L2 of the GPU output against it, as is and with
    bf16 rounding ties forgiven: a one-ulp bf16 difference where the
    oracle's fp32 value lies within 2^-16 of the two values' midpoint), and
    the fp64 exact attention of the bf16 inputs gives the cosines of both."""
    import numpy as np
    import oracle
    Nq, N = q.shape[2], k.shape[2]
    nqb = (Nq + 127) // 128
    rng = np.random.default_rng(1)
    units = sorted({(0, 0), (w.B * w.H - 1, nqb - 1)} |
                   {(int(rng.integers(w.B * w.H)), int(rng.integers(nqb))) for _ in range(nunits - 2)})
    heads = sorted({bh for bh, _ in units})
    pos = {bh: i for i, bh in enumerate(heads)}
    sub = [(pos[bh], qb) for bh, qb in units]

    def hd(t):
        B, H, n, d = t.shape
        return t.reshape(B * H, n, d)[heads].reshape(1, len(heads), n, d).contiguous()
    qs, ks, vs = hd(q), hd(k), hd(v)
    rq = oracle.quantize_qkv(qs, ks, vs, smooth_v=vsm)
    ref32 = np.zeros((1, len(heads), Nq, w.d), np.float32)
    ref = oracle.bf16_bits_to_f32(oracle.attn_fwd(rq, Nq, causal, units=sub, p_two_level=two, out32=ref32))[0]
    ref32 = ref32[0]
    ex = oracle.attn_exact(qs, ks, vs, causal, units=sub)[0]
    got = out.float().cpu().numpy().reshape(w.B * w.H, Nq, w.d)[heads]
    live = (np.arange(Nq) + (N - Nq) >= 0) if causal else np.ones(Nq, bool)
    def tied(g, r, r32):
        # adjacent bf16 values of one sign whose fp32 source sits on their midpoint
        gb = (np.ascontiguousarray(g, np.float32).view(np.uint32) >> 16).astype(np.int64)
        rb = (np.ascontiguousarray(r, np.float32).view(np.uint32) >> 16).astype(np.int64)
        mid = (g.astype(np.float64) + r.astype(np.float64)) / 2
        return (np.abs(gb - rb) == 1) & ((gb >> 15) == (rb >> 15)) & \
            (np.abs(r32.astype(np.float64) - mid) <= 2.0 ** -16 * np.abs(mid))
    worst, worst_t, gs, rs, es = 0.0, 0.0, [], [], []
    for h, qb in sub:
        rows = np.arange(qb * 128, min(Nq, qb * 128 + 128))
        rows = rows[live[rows]]
        if rows.size == 0:
            continue
        g, r, e = (a[h, rows].astype(np.float64) for a in (got, ref, ex))
        worst = max(worst, float(np.linalg.norm(g - r) / np.linalg.norm(r)))
        gt = np.where(tied(got[h, rows], ref[h, rows], ref32[h, rows]), r, g)
        worst_t = max(worst_t, float(np.linalg.norm(gt - r) / np.linalg.norm(r)))
        gs.append(g.ravel())
        rs.append(r.ravel())
        es.append(e.ravel())
    g, r, e = np.concatenate(gs), np.concatenate(rs), np.concatenate(es)

    def cos(a, b):
        return float(a @ b / np.sqrt((a @ a) * (b @ b)))
    return {"rel_l2_vs_oracle_worst_block": float(f"{worst:.3e}"),
            "rel_l2_vs_oracle_worst_block_ties_forgiven": float(f"{worst_t:.3e}"),
            "cosine_vs_exact": round(cos(g, e), 5),
            "oracle_cosine_vs_exact": round(cos(r, e), 5),
            "sample": f"{len(units)} (head, 128-row Q block) units; the oracle quantizes those heads itself"}


def attn_ops(w, Nq):
    """4*d per visible (query, key) pair: the workload's own count (4*B*H*N^2*d,
    halved for causal) when Nq == N, else the exact count of pairs that the
    mask leaves (causal: query r sees keys 0 .. r + N - Nq)."""
    if Nq == w.N:
        return w.ops
    if not w.causal:
        return 4.0 * w.B * w.H * Nq * w.N * w.d
    off = w.N - Nq
    pairs = sum(min(max(r + off + 1, 0), w.N) for r in range(Nq))
    return 4.0 * w.B * w.H * pairs * w.d


def processed_s_elements(B, H, Nq, N, causal):
    """S elements the attention kernels compute: whole 128 x 128 tiles, for
    each Q tile the KV blocks up to the one holding its last row's diagonal
    (causal; the last query lines up with the last key), all of them else."""
    nqt, nkvt, off = (Nq + 127) // 128, (N + 127) // 128, N - Nq
    total = 0
    for t in range(nqt):
        last = t * 128 + 127 + off
        total += min(last // 128 + 1, nkvt) if (causal and last >= 0) else (0 if causal else nkvt)
    return B * H * total * 128 * 128


def exp2_ceiling_us(B, H, Nq, N, causal, sm_mhz, n_sm):
    """Time the FP4 attention kernel would take if its exp2 unit were busy
    every cycle: EX2_PER_S exponentials per computed S element at
    EX2_PER_SM_CLK per SM per clock, at the sampled SM clock."""
    n = processed_s_elements(B, H, Nq, N, causal) * EX2_PER_S
    return n / (EX2_PER_SM_CLK * n_sm * sm_mhz * 1e6) * 1e6


def make_inputs(w, Nq, seed):
    """The workload's seeded q, k, v; q cut to (or drawn with) Nq tokens."""
    if Nq <= w.N:
        q, k, v = sa3_inputs.make_qkv(w, seed=seed)
        return (q[:, :, :Nq].contiguous() if Nq < w.N else q), k, v
    q, k, v = sa3_inputs.make_qkv(w, seed=seed, shape_override={"N": Nq})
    return q, k[:, :, :w.N].contiguous(), v[:, :, :w.N].contiguous()


def run_sa3(args, rank, world, local):
    import bit_quantized_attention_sa3_b200 as sa3
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = sa3_inputs.WORKLOADS[args.workload]
    B, H, N, d, causal = w.B, w.H, w.N, w.d, w.causal
    Nq = args.nq or N
    two = bool(args.p_two_level)
    vsm = bool(args.v_smooth)
    qload = bool(args.q_on_load)
    q_h, k_h, v_h = make_inputs(w, Nq, seed=rank)
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    i8 = args.variant in ("i8", "i8_train")
    train = args.variant == "i8_train"
    if i8:
        empty_q, quantize = sa3.empty_quantized_i8, sa3.quantize_qkv_i8
    else:
        def empty_q(B, H, N, d, dev, Nq):
            return sa3.empty_quantized(B, H, N, d, dev, Nq=Nq, v_smooth=vsm, skip_q=qload)

        def quantize(q, k, v, out, workspace, stream=None):
            return sa3.quantize_qkv(q, k, v, out=out, workspace=workspace, stream=stream, v_smooth=vsm,
                                    skip_q=qload)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=dev) if train else None

    def attend(qz, causal, out, stream=None, lse=lse, qsrc=None):
        if i8:
            return sa3.attn_fwd_i8(qz, causal=causal, out=out, stream=stream, lse=lse)
        return sa3.attn_fwd(qz, causal=causal, out=out, stream=stream, p_two_level=two,
                            q=qsrc if qload else None)
    qz = empty_q(B, H, N, d, dev, Nq=Nq)
    ws = torch.empty(max(16, sa3.quant_workspace_bytes(B, H, N, d, vsm)), dtype=torch.uint8, device=dev)
    out = torch.empty((B, H, Nq, d), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    clean = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    clean_sum = torch.empty((), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def flush_l2(i):
        flush.fill_(i & 0xFF)                # evict everything the previous step left in L2
        torch.sum(clean, dim=0, out=clean_sum)  # refill L2 with clean, unrelated lines

    def step():
        quantize(q, k, v, out=qz, workspace=ws)
        attend(qz, causal=causal, out=out, qsrc=q)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if sa3.device_status() != sa3.SA3_OK:
        raise RuntimeError("device wait gave up during warm-up")

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    with ClockSampler(local) as clk:
        time.sleep(0.01)  # first sample before the timed region starts
        # one more untimed step: the GPU sat idle during the sleep, and the
        # first step after an idle spell runs slow (131 us instead of 36 us
        # for the quantizer on the headline shape)
        flush_l2(args.steps)
        step()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)
        for i in range(args.steps):
            flush_l2(i)
            ev[i][0].record(stream)
            quantize(q, k, v, out=qz, workspace=ws)
            ev[i][1].record(stream)
            attend(qz, causal=causal, out=out, qsrc=q)
            ev[i][2].record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            torch.distributed.barrier()
    step_ms = [ev[i][0].elapsed_time(ev[i][2]) for i in range(args.steps)]
    quant_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(args.steps)]
    attn_ms = [ev[i][1].elapsed_time(ev[i][2]) for i in range(args.steps)]
    if sa3.device_status() != sa3.SA3_OK:
        raise RuntimeError("device wait gave up during the timed steps")

    # end-to-end through the public API: pinned host in -> host out, every
    # step copying its inputs up and its output down.  Pipelined as a serving
    # loop would run it: two buffer sets, uploads on one stream, kernels on
    # the launching stream, downloads on a third, so that step i+1's upload
    # and step i-1's download overlap step i's kernels.
    qp, kp, vp = q_h.pin_memory(), k_h.pin_memory(), v_h.pin_memory()
    up_s, down_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    sets = []
    for _ in range(2):
        sets.append(dict(q=torch.empty_like(q), k=torch.empty_like(k), v=torch.empty_like(v),
                         qz=empty_q(B, H, N, d, dev, Nq=Nq), ws=torch.empty_like(ws),
                         out=torch.empty_like(out),
                         out_h=torch.empty((B, H, Nq, d), dtype=torch.bfloat16).pin_memory(),
                         lse=torch.empty_like(lse) if train else None,
                         lse_h=torch.empty((B, H, Nq), dtype=torch.float32).pin_memory() if train else None,
                         ready=torch.cuda.Event(), done=torch.cuda.Event(), free=torch.cuda.Event()))

    def e2e_run(n):
        for i in range(n):
            b = sets[i % 2]
            if i >= 2:
                up_s.wait_event(b["free"])      # step i-2 has consumed and returned this set
            with torch.cuda.stream(up_s):
                b["q"].copy_(qp, non_blocking=True)
                b["k"].copy_(kp, non_blocking=True)
                b["v"].copy_(vp, non_blocking=True)
                b["ready"].record(up_s)
            stream.wait_event(b["ready"])
            quantize(b["q"], b["k"], b["v"], out=b["qz"], workspace=b["ws"], stream=stream)
            attend(b["qz"], causal=causal, out=b["out"], stream=stream, lse=b["lse"], qsrc=b["q"])
            b["done"].record(stream)
            down_s.wait_event(b["done"])
            with torch.cuda.stream(down_s):
                b["out_h"].copy_(b["out"], non_blocking=True)
                if train:
                    b["lse_h"].copy_(b["lse"], non_blocking=True)
                b["free"].record(down_s)
        stream.wait_stream(up_s)
        stream.wait_stream(down_s)

    e2e_run(max(2, args.warmup // 2))
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = max(3, args.steps // 2)
    if world > 1:
        torch.distributed.barrier()
    e0.record(stream)
    e2e_run(n_e2e)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / n_e2e
    if not torch.equal(sets[(n_e2e - 1) % 2]["out_h"], out.cpu()):
        raise RuntimeError("end-to-end output differs from the device-resident run")
    if train and not torch.equal(sets[(n_e2e - 1) % 2]["lse_h"], lse.cpu()):
        raise RuntimeError("end-to-end log-sum-exp differs from the device-resident run")

    def gmax(x):
        if world == 1:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        return float(t.item())

    probe = None if i8 else fp4_peak_probe(sa3, dev)
    t_step = gmax(sum(step_ms) / len(step_ms))
    t_quant = gmax(sum(quant_ms) / len(quant_ms))
    t_attn = gmax(sum(attn_ms) / len(attn_ms))
    t_e2e = gmax(e2e_ms)
    if rank != 0:
        return
    pk, src = peaks()
    ops = attn_ops(w, Nq)
    achieved = ops / (t_attn * 1e-3) / 1e12
    Np, Npq = sa3.padded_len(N), sa3.padded_len(Nq)
    nq_quant = 0 if qload else Nq               # Q on load: the quantizer reads and writes no Q
    rd = B * H * d * 2 * (nq_quant + 2 * N)     # bf16 q, k, v read once
    if i8:
        # half the ops at the int8 rate (2x bf16, nominal), half at the fp16 rate
        peak = pk["bf16_tflops"] * 4.0 / 3.0
        peak_src = f"{src} bf16 burst {pk['bf16_tflops']} x 4/3 (QK^T at the nominal int8 rate 2x, P V at 1x)"
        qk_bytes = rd + B * H * d * (Npq + Np) + B * H * d * Np * 2 + B * H * ((Npq + Np) // 128) * 4
        dtype = "int8 QK^T (fp32 scale per 128-token tile), fp16 P V, fp32 accumulate"
        kernel, traffic = "attn8_fwd_kernel<%d>" % d, None
    else:
        peak = probe["tops"]
        peak_src = (f"measured in this run: {probe['how']} (N=128 {probe['n128_tops']}, "
                    f"N=256 {probe['n256_tops']} TOPS)")
        peak_rule = pk["bf16_tflops"] * FP4_PER_BF16
        npq_quant = 0 if qload else Npq
        qk_bytes = rd + B * H * d * (npq_quant + 2 * Np) // 2 + B * H * d * (npq_quant + 2 * Np) // 16
        dtype = "fp4-e2m1 (ue4m3 scales, fp32 accumulate)"
        kernel = "attn_fwd_kernel<%d>" % d
        traffic = profiled_traffic("bit_quantized_attention_sa3_b200/csrc/attn.cuh",
                                   "attn_fwd_kernel_d128_noncausal_b2h16n4096d128.md") \
            if (d, args.workload, Nq, two) == (128, WORKLOAD, N, False) else None
    line = {
        "metric": METRIC,
        "value": round(world * ops / (t_step * 1e-3) / 1e12, 2),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(t_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": dtype,
        "data": "synthetic (seeded, sa3_inputs.py)",
        "config": {"workload": w.name, "B": B, "H": H, "N": N, "d": d, "causal": causal,
                   "variant": args.variant,
                   "step": ("sa3_quantize_qkv_i8 + sa3_attn_fwd_i8_lse" if train else
                            "sa3_quantize_qkv_i8 + sa3_attn_fwd_i8" if i8 else "sa3_quantize_qkv + sa3_attn_fwd"),
                   "l2": "flushed before each step: 256 MiB write, then 256 MiB read of another buffer",
                   "parallelism": f"{world} independent replicas (one batch per GPU)"},
        "attn_only": {"value": round(achieved, 2), "unit": UNIT, "ms": round(t_attn, 4),
                      "frac_of_datasheet_fp4_9000": round(achieved / FP4_DATASHEET_TOPS, 4)},
        "quantize": {"ms": round(t_quant, 4), "GB_per_s": round(qk_bytes / (t_quant * 1e-3) / 1e9, 1),
                     "algorithmic_bytes": qk_bytes},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": round(peak, 1),
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "traffic": traffic,
                     "kernel": kernel, "peak_source": peak_src},
        "e2e": {"value": round(world * ops / (t_e2e * 1e-3) / 1e12, 2), "unit": UNIT, "ms": round(t_e2e, 4),
                "pipelined": "2 buffer sets; upload, kernels and download on three streams",
                "h2d_bytes_per_step": rd,
                "d2h_bytes_per_step": B * H * Nq * d * 2 + (B * H * Nq * 4 if train else 0)},
        "gpu_launches": LAUNCHES_PER_STEP * args.steps,
        "clocks": clk.summary(),
    }
    if not i8:
        line["roofline"]["peak_bf16x4"] = round(peak_rule, 1)
        line["roofline"]["frac_of_bf16x4"] = round(achieved / peak_rule, 4)
        line["roofline"]["peak_bf16x4_source"] = f"{src} bf16 burst {pk['bf16_tflops']} x 4 (nominal FP4/bf16 ratio)"
        try:  # the kernel's binding limit: its exponentials (never fails the line)
            mhz = line["clocks"].get("sm_mhz") or line["clocks"].get("sm_max_mhz")
            n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
            ceil_us = exp2_ceiling_us(B, H, Nq, N, causal, float(mhz), n_sm)
            line["roofline"]["exp2_ceiling"] = {
                "us": round(ceil_us, 1), "frac": round(ceil_us / (t_attn * 1e3), 4),
                "how": (f"{EX2_PER_S:.4f} ex2 per computed S element (whole 128x128 tiles) at "
                        f"{EX2_PER_SM_CLK} per SM per clock, {n_sm} SMs, {mhz} MHz")}
        except Exception as e:  # noqa: BLE001
            line["roofline"]["exp2_ceiling"] = {"us": None, "error": repr(e)[:120]}
    if Nq != N:
        line["config"]["Nq"] = Nq
        line["config"]["ops"] = "4*d per (query, key) pair the mask leaves"
    if two:
        line["config"]["p_two_level"] = True
    if vsm:
        line["config"]["v_smooth"] = True
    if qload:
        line["config"]["q_on_load"] = True
        line["config"]["step"] = "sa3_quantize_qkv_ex (SA3_SKIP_Q) + sa3_attn_fwd_ex (SA3_Q_ON_LOAD)"
    if world == 1 and not args.skip_cpu_baseline:
        if not i8:
            line["accuracy"] = accuracy_sample(w, q_h, k_h, v_h, out, causal, two=two, vsm=vsm)
        line["cpu_baseline"] = cpu_baseline(w, q_h, k_h, v_h, budget_s=15.0, i8=i8, train=train, two=two, vsm=vsm)
    print(json.dumps(line), flush=True)


def cpu_baseline(w, q, k, v, budget_s=15.0, units_cap=None, i8=False, train=False, two=False, vsm=False):
    """The oracle, as it stands, on the host cores: full quantization plus
    attention for a seeded sample of Q blocks; the full-job time is
    extrapolated from the sampled blocks, each weighted by the KV blocks it
    processes (non-causal: all the same)."""
    import numpy as np
    import oracle
    oracle.build()
    Nq, N = q.shape[2], k.shape[2]
    t0 = time.perf_counter()
    qz = oracle.quantize_qkv_i8(q, k, v) if i8 else oracle.quantize_qkv(q, k, v, smooth_v=vsm)
    t_quant = time.perf_counter() - t0
    nqb, nkv = (Nq + 127) // 128, (N + 127) // 128
    total_units = w.B * w.H * nqb
    rng = np.random.default_rng(0)
    order = rng.permutation(total_units)
    done, t_attn, n = 0, 0.0, 8
    while True:
        chunk = order[done:done + n]
        if len(chunk) == 0:
            break
        units = [(int(u) // nqb, int(u) % nqb) for u in chunk]
        t0 = time.perf_counter()
        if i8:
            oracle.attn_fwd_i8(qz, Nq, w.causal, units=units, return_lse=train)
        else:
            oracle.attn_fwd(qz, Nq, w.causal, units=units, p_two_level=two)
        t_attn += time.perf_counter() - t0
        done += len(chunk)
        if t_quant + t_attn > budget_s or (units_cap and done >= units_cap):
            break
        n = min(4 * n, 256)
    if w.causal:
        last = np.arange(nqb) * 128 + 127 + (N - Nq)
        per_tile = np.clip(np.where(last < 0, 0, last // 128 + 1), 0, nkv).astype(float)
        weights = per_tile[np.arange(total_units) % nqb]
        frac = weights[order[:done]].sum() / max(weights.sum(), 1.0)
    else:
        frac = done / total_units
    t_full = t_quant + t_attn / frac
    return {"value": round(attn_ops(w, Nq) / t_full / 1e12, 6), "unit": UNIT, "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": (f"full quantization ({t_quant:.2f} s) + attention for {done} of {total_units} "
                       f"Q blocks ({t_attn:.2f} s), extrapolated to the whole {w.name} job "
                       f"({t_full:.1f} s)")}


def run_reference(args, rank, world):
    if rank != 0:
        return
    w = sa3_inputs.WORKLOADS[args.workload]
    Nq = args.nq or w.N
    q, k, v = make_inputs(w, Nq, seed=0)
    per_step, wall = [], []
    budget = max(5.0, 150.0 / max(1, args.steps + args.warmup))
    i8, train = args.variant in ("i8", "i8_train"), args.variant == "i8_train"
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        cb = cpu_baseline(w, q, k, v, budget_s=budget, i8=i8, train=train, two=bool(args.p_two_level),
                          vsm=bool(args.v_smooth))
        if i >= args.warmup:
            per_step.append(cb)
            wall.append(time.perf_counter() - t0)
    vals = [c["value"] for c in per_step]
    value = statistics.mean(vals)
    last = per_step[-1]
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(attn_ops(w, Nq) / (value * 1e12) * 1e3, 3),
        "ms_per_step_kind": ("extrapolated: the time the oracle would take for one whole step, from full "
                             "quantization plus a timed sample of Q blocks; each sampled step took "
                             "sampled_ms_per_step of wall time"),
        "sampled_ms_per_step": round(1e3 * statistics.mean(wall), 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64/f32 (CPU oracle)",
        "data": "synthetic (seeded, sa3_inputs.py)",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal,
                   "variant": args.variant, **({"Nq": Nq} if Nq != w.N else {}),
                   **({"p_two_level": True} if args.p_two_level else {}),
                   **({"v_smooth": True} if args.v_smooth else {}),
                   "step": "oracle quantize + tiled attention (sampled, extrapolated)"},
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": last["cores"], "kind": "oracle",
                         "sample": last["sample"]},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank, world, local = dist_init(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_sa3(args, rank, world, local)
    finally:
        if world > 1 and torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
