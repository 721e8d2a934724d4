"""Benchmark: block-causal attention forward + JVP on B200.

One step = one call of the fused kernel over the whole workload (every head of
every batch entry), inputs resident in HBM. Default workload: the teacher-forcing
frame-wise Wan2.1-1.3B-shaped layout (B=1, H=12, D=128, 21 clean + 21 noisy
latent frames of 1560 tokens, N=65520, bf16 in / fp32 accumulate). The default
single-GPU run also times the other four workloads (one key each under
"configs"), the backward, the prologue, the output projection, the
clean-tangent-zero call and the context-parallel scatter.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--split tiles|heads|replicas|ulysses] [--fused-output]

Prints one JSON line on rank 0. Multi-GPU runs (torchrun) split one problem:
by default its 128-row query tiles are dealt out to the ranks by cost, every
rank holding the whole inputs and running its tiles for every head
(independent problems, no data-path collective, strong scaling); --split heads
gives every rank whole heads; --split ulysses gives every rank a sequence shard
and runs the Ulysses all-to-all path; --split replicas gives every rank its own
copy (weak scaling). Throughput is whole-job work over the slowest rank's time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from masked_attention_jvp_b200.workloads import WORKLOADS, BENCH_WORKLOAD, make_inputs  # noqa: E402

METRIC = "block-causal attention fwd+JVP TFLOP/s and % of B200 dense BF16 peak"
DENSE_BF16_SPEC_TFLOPS = 2250.0
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}


# DRAM bytes per launch of the tensor-core kernel on the TF frame-wise workload,
# from one ncu capture (dram__bytes_read.sum + dram__bytes_write.sum), keyed by a
# hash of the kernel sources it was taken on: a changed kernel reports null.
# each kernel's sources plus the parameter struct it is launched with
KERNEL_SOURCES = ["fwd_jvp_sm100.cu", "ptx_sm100.cuh", "mask_schedule.h", "struct Sm100Params"]
PROLOGUE_SOURCES = ["prologue.cu", "struct PrologueParams"]
BACKWARD_SOURCES = ["bwd_sm100.cu", "ptx_sm100.cuh", "mask_schedule.h", "struct BwdParams"]
OUT_PROJ_SOURCES = ["out_proj_sm100.cu", "ptx_sm100.cuh", "struct OutProjParams"]
# {(workload, code hash of the kernel's sources): dram bytes read + written per launch}
MEASURED_TRAFFIC = {("wan1.3b_tf_framewise", "97b5a02ae04b9fdf"): 1425837824 + 391129344}
PROLOGUE_TRAFFIC = {("wan1.3b_tf_framewise", "34494554b0571872"): 1241276160 + 1150380544}
# one launch of the output projection on the workload's tokens (M = 65520, K = C = 1536)
OUT_PROJ_TRAFFIC = {("wan1.3b_tf_framewise", "f7d2c6975f9ce8cc"): 407364608 + 365617152}
# summed over the three launches of one backward call (delta, dQ, dK/dV)
BACKWARD_TRAFFIC = {("wan1.3b_tf_framewise", "07580bab5d2f1875"):
                    402566144 + 5953792 + 814209024 + 184451328 + 816486656 + 383889664}


def _code_only(text: str) -> str:
    """The code of a C/CUDA source: comments removed, whitespace runs collapsed,
    so that editing a comment does not invalidate measured counters."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_sources_hash(files=KERNEL_SOURCES, read=None) -> str:
    """sha256 prefix over the code (not the comments) of a kernel's sources and
    its parameter struct. `read(name)` returns a file of csrc/ as text (default:
    the working tree)."""
    import hashlib
    import re
    csrc = os.path.join(ROOT, "masked_attention_jvp_b200", "csrc")
    if read is None:
        def read(name):
            with open(os.path.join(csrc, name), encoding="utf-8") as fh:
                return fh.read()
    h = hashlib.sha256()
    for f in files:
        if f.startswith("struct "):
            m = re.search(r"^%s \{.*?^\};" % re.escape(f), read("kernels.h"), re.S | re.M)
            h.update(_code_only(m.group(0) if m else f).encode())
        else:
            h.update(_code_only(read(f)).encode())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def workload_config(w, extra=None):
    m = w.mask
    cfg = {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "D": w.D,
           "tokens_per_frame": m.tokens_per_frame, "frames_per_chunk": m.frames_per_chunk,
           "n_frames": m.n_frames, "tf_layout": m.tf_layout,
           "dtype_in": str(w.dtype).split(".")[-1], "accumulate": "fp32",
           "l2": "inputs larger than L2 (6 bf16 tensors of %.2f GB total per step)" % (
               6 * w.B * w.H * w.N * w.D * 2 / 1e9)}
    if extra:
        cfg.update(extra)
    return cfg


def flops_of(w):
    from masked_attention_jvp_b200 import flops
    return flops(w.B, w.H, w.D, w.mask)


def ctz_product_flops(w):
    """Products actually needed when clean tangents vanish (teacher forcing):
    clean rows 2 products per visible pair (S, PV), noisy rows over clean keys
    4 (S, tQ K^T, PV, (P o tS) V), noisy rows over their own chunk all 6; each
    product is 2 D flops per pair."""
    m = w.mask
    G, n = m.frames_per_chunk * m.tokens_per_frame, m.n_frames // m.frames_per_chunk
    clean = G * G * n * (n + 1) // 2
    noisy_clean = G * G * n * (n - 1) // 2
    noisy_own = G * G * n
    return 2 * w.D * (2 * clean + 4 * noisy_clean + 6 * noisy_own) * w.B * w.H


# ----------------------------------------------------------------- CPU oracle
def oracle_rows_flops(w, rows):
    """12 D flops per visible key of each sampled row (same count as the GPU)."""
    import oracle
    m = w.mask
    G, L = m.frames_per_chunk * m.tokens_per_frame, m.n_frames * m.tokens_per_frame
    total = 0
    for r in rows.tolist():
        i = r % w.N
        if not m.tf_layout or i < L:
            nk = (i // G + 1) * G
        else:
            nk = ((i - L) // G) * G + G
        total += nk
    return 12 * w.D * total


def time_oracle(w, target_s=15.0, host_inputs=None):
    """Times the oracle as it stands on a bounded row sample of workload `w`.
    Returns (TFLOP/s, seconds, rows, threads, description)."""
    import oracle
    from masked_attention_jvp_b200.workloads import sample_rows
    ins = host_inputs if host_inputs is not None else make_inputs(w, "cpu")
    threads = oracle.max_threads()
    per_head = 4
    rows = sample_rows(w, per_head, seed_offset=77)
    t0 = time.perf_counter()
    oracle.attn_fwd_jvp_rows(*ins, w.mask, scale=w.scale, rows=rows)
    dt = time.perf_counter() - t0
    # scale the sample to about target_s seconds of CPU work
    per_head = max(1, min(w.N, int(per_head * target_s / max(dt, 1e-3))))
    rows = sample_rows(w, per_head, seed_offset=78)
    t0 = time.perf_counter()
    oracle.attn_fwd_jvp_rows(*ins, w.mask, scale=w.scale, rows=rows)
    dt = time.perf_counter() - t0
    fl = oracle_rows_flops(w, rows)
    desc = (f"{rows.numel()} seeded query rows ({per_head} per head x {w.B * w.H} heads) of "
            f"{w.name}, fp64 oracle, {threads} OpenMP threads")
    return fl / dt / 1e12, dt, rows.numel(), threads, desc


def host_cpu() -> dict:
    """The host CPU's model name and logical core count (for the oracle baseline)."""
    model = None
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return {"model": model, "nproc": os.cpu_count()}


# ------------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event reasons of this process's GPU, sampled every
    10 ms through NVML while the `with` block runs (reads only; nothing is set).
    Falls back to `nvidia-smi -lms 100` where NVML is unavailable."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4}

    def __init__(self, cuda_index: int, period_s: float = 0.01):
        self.cuda_index = cuda_index
        self.period = period_s
        self.rows = []          # (sm_mhz, max_mhz, reasons bitmask)
        self.nvml = None
        self.thread = None
        self.stop = None
        self.proc = None
        self.path = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        self.nvml = pynvml
        props = torch.cuda.get_device_properties(self.cuda_index)
        bus = getattr(props, "pci_bus_id", None)
        if bus is not None:
            pci = f"{getattr(props, 'pci_domain_id', 0):08x}:{bus:02x}:{getattr(props, 'pci_device_id', 0):02x}.0"
            try:
                return pynvml.nvmlDeviceGetHandleByPciBusId(pci)
            except pynvml.NVMLError:
                pass
        return pynvml.nvmlDeviceGetHandleByIndex(self.cuda_index)

    def _sample(self, h):
        nv = self.nvml
        max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        while not self.stop.is_set():
            try:
                self.rows.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM), max_mhz,
                                  nv.nvmlDeviceGetCurrentClocksEventReasons(h)))
            except nv.NVMLError:
                return
            self.stop.wait(self.period)

    def __enter__(self):
        import threading
        try:
            h = self._nvml_handle()
            self.stop = threading.Event()
            self.thread = threading.Thread(target=self._sample, args=(h,), daemon=True)
            self.thread.start()
            return self
        except Exception:
            self.nvml = None
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.cuda_index}", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
            try:
                self.nvml.nvmlShutdown()
            except Exception:
                pass
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            names = list(self.REASONS)
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    mask = sum(self.REASONS[n] for n, v in zip(names, parts[5:9]) if v == "Active")
                    self.rows.append((float(parts[1]), float(parts[2]), mask))
                except ValueError:
                    continue
            os.unlink(self.path)

    def summary(self):
        if not self.rows:
            return None
        reasons = sorted(n for n, bit in self.REASONS.items() if any(r[2] & bit for r in self.rows))
        return {"sm_mhz": statistics.median(r[0] for r in self.rows), "sm_max_mhz": max(r[1] for r in self.rows),
                "reasons": reasons, "samples": len(self.rows),
                "source": "nvml, 10 ms" if self.nvml is not None else "nvidia-smi, 100 ms"}


# ------------------------------------------------------------- multi-rank
def max_over_ranks(value: float, world: int, device) -> float:
    """Slowest rank's time: an all-reduce MAX of one scalar (the only
    collective of the benchmark; none sits on the data path)."""
    if world <= 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_rank: int, world: int, steps: int, slowest_ms: float) -> float:
    """Whole-job throughput: every rank processes its own copy of the workload
    (weak scaling), all of them within the slowest rank's time."""
    return world * flops_per_rank * steps / (slowest_ms / 1e3) / 1e12


def split_heads(H: int, world: int, rank: int):
    """Heads [h0, h1) of `rank` when one problem's H heads are spread over
    `world` ranks as evenly as they go (the first H % world ranks take one
    more). Heads are independent problems, so no collective joins them."""
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def strong_tflops(total_flops: int, steps: int, slowest_ms: float) -> float:
    """Whole-job throughput of one problem split over the ranks (strong
    scaling): the whole problem's work per step, done within the slowest
    rank's time."""
    return total_flops * steps / (slowest_ms / 1e3) / 1e12


# ------------------------------------------------------------------ prologue
def bench_prologue(w, dev, steps, peaks):
    """The attention block's prologue in primal-tangent form (QK-RMSNorm + JVP,
    rotary embedding, re-layout of all six tensors) on the workload's shape:
    HBM-bound, reported against the measured copy bandwidth."""
    import masked_attention_jvp_b200 as caj
    B, N, H, D = w.B, w.N, w.H, w.D
    C = H * D
    g = torch.Generator(device=dev).manual_seed(w.seed)
    xs = [torch.randn(B, N, C, device=dev, generator=g).to(torch.bfloat16) for _ in range(6)]
    gq = torch.ones(C, device=dev)
    gk = torch.ones(C, device=dev)
    inv = 10000.0 ** (-torch.arange(0, D, 2, device=dev, dtype=torch.float32) / D)
    ang = torch.arange(N, device=dev, dtype=torch.float32)[:, None] * inv[None, :]
    cos, sin = torch.cos(ang).contiguous(), torch.sin(ang).contiguous()
    out = [torch.empty(B, H, N, D, dtype=torch.bfloat16, device=dev) for _ in range(6)]
    for _ in range(3):
        caj.qk_norm_rope_jvp(*xs, gq, gk, cos, sin, H, out=out)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        caj.qk_norm_rope_jvp(*xs, gq, gk, cos, sin, H, out=out)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    algo = 12 * B * N * C * 2 + 2 * N * (D // 2) * 4 + 2 * C * 4
    gbs = algo / (ms / 1e3) / 1e9
    peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    return {"kernel": "qk_norm_rope_jvp_kernel<%d>" % D, "shape": [B, N, H, D], "ms": round(ms, 4),
            "bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
            "frac": round(gbs / peak, 4), "algorithmic_bytes": algo,
            "traffic": PROLOGUE_TRAFFIC.get((w.name, kernel_sources_hash(PROLOGUE_SOURCES))),
            "note": "inputs 6 x [B,N,H*D] + outputs 6 x [B,H,N,D] bf16 > L2"}


# ------------------------------------------------------------------ backward
def bench_backward(w, ins, o, lse, steps, peaks):
    """Backward of the primal attention (delta pre-pass, dQ kernel, dK/dV kernel)
    on the same workload. Algorithmic work: the five products of the standard
    count, 10 D flops per visible pair per head (the kernels recompute S and dP
    once more, 14 D in total)."""
    import masked_attention_jvp_b200 as caj
    q, k, v = ins[:3]
    g = torch.Generator(device=q.device).manual_seed(w.seed + 1)
    dout = torch.randn(q.shape, device=q.device, generator=g).to(torch.bfloat16)
    for _ in range(3):
        caj.attn_bwd(q, k, v, o, dout, lse, w.mask, scale=w.scale)
    torch.cuda.synchronize()
    caj.device_status()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        caj.attn_bwd(q, k, v, o, dout, lse, w.mask, scale=w.scale)
    e1.record()
    torch.cuda.synchronize()
    caj.device_status()
    ms = e0.elapsed_time(e1) / steps
    pairs = flops_of(w) // (12 * w.D)
    alg = 10 * w.D * pairs
    tf = alg / (ms / 1e3) / 1e12
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    return {"kernels": ["bwd_delta_kernel", "bwd_dq_kernel", "bwd_dkdv_kernel"], "ms": round(ms, 4),
            "bound": "tensor", "achieved": round(tf, 2), "peak": peak, "unit": "TFLOP/s",
            "frac": round(tf / peak, 4), "flop_count": "10*D per visible pair (5 products)",
            "traffic": BACKWARD_TRAFFIC.get((w.name, kernel_sources_hash(BACKWARD_SOURCES))),
            "executed_products_tflop": round(14 * w.D * pairs / 1e12, 3)}


# ------------------------------------------------- clean-tangent-zero forward
def bench_ctz(w, ins, steps, fl):
    """The same workload as TF-sCM feeds it: the clean half's tangents are zero
    and the call skips the products that vanish (two launches per call). The
    value is dense-equivalent (12 D flops per visible pair) and, separately,
    per needed product."""
    import masked_attention_jvp_b200 as caj
    from masked_attention_jvp_b200.workloads import zero_clean_tangents
    tq, tk, tv = (t.clone() for t in ins[3:])
    zero_clean_tangents(w, tq, tk, tv)
    args = ins[:3] + [tq, tk, tv]
    o, to = torch.empty_like(ins[0]), torch.empty_like(ins[0])
    lse = torch.empty(ins[0].shape[:3], dtype=torch.float32, device=ins[0].device)
    tlse = torch.empty_like(lse)

    def call():
        caj.attn_fwd_jvp_out(*args, w.mask, o, to, lse, tlse, scale=w.scale, clean_tangent_zero=True)
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        call()
    e1.record()
    torch.cuda.synchronize()
    caj.device_status()
    ms = e0.elapsed_time(e1) / steps
    L = w.mask.n_frames * w.mask.tokens_per_frame
    return {"ms": round(ms, 4), "dense_equivalent_tflops": round(fl / (ms / 1e3) / 1e12, 2),
            "needed_products_tflop": round(ctz_product_flops(w) / 1e12, 3),
            "needed_products_tflops": round(ctz_product_flops(w) / (ms / 1e3) / 1e12, 2),
            "kernels": ["fwd_jvp_sm100_kernel<128, kTilesNoisyCTZ>", "fwd_primal_sm100_kernel<128>"],
            "gpu_launches": steps * (2 if L >= 128 else 1)}


# ------------------------------------------------------------ output projection
def bench_out_proj(w, dev, steps, peaks):
    """Output projection in primal-tangent form on the workload's tokens:
    y = x W^T + b, ty = tx W^T with x, tx [B*N, H*D] and W [H*D, H*D] (the
    model width; Wan-1.3B: 1536), 2*M*K*C flops each, in one launch of the
    library's kernel. PyTorch's cuBLAS matmuls on the same tensors are timed
    beside it as a library reference."""
    import masked_attention_jvp_b200 as caj
    M, K = w.B * w.N, w.H * w.D
    C = K
    g = torch.Generator(device=dev).manual_seed(w.seed + 3)
    x, tx = (torch.randn(M, K, device=dev, generator=g).to(torch.bfloat16) for _ in range(2))
    wt = (torch.randn(C, K, device=dev, generator=g) / K ** 0.5).to(torch.bfloat16)
    b = torch.randn(C, device=dev, generator=g).to(torch.bfloat16)
    out = (torch.empty(M, C, device=dev, dtype=torch.bfloat16), torch.empty(M, C, device=dev, dtype=torch.bfloat16))

    def ours():
        caj.out_proj_jvp(x, tx, wt, b, out=out)

    def cublas():
        torch.addmm(b, x, wt.t(), out=out[0])
        torch.mm(tx, wt.t(), out=out[1])

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    # alternate, so that clock drift under the power cap affects both alike
    t_ours, t_lib = [], []
    for _ in range(2):
        t_ours.append(timed(ours))
        t_lib.append(timed(cublas))
    caj.device_status()
    ms, ms_lib = min(t_ours), min(t_lib)
    fl = 2 * 2 * M * K * C
    tf = fl / (ms / 1e3) / 1e12
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    return {"op": "y = x W^T + b, ty = tx W^T (out_proj_sm100_kernel, one launch)", "M": M, "K": K, "C": C,
            "ms": round(ms, 4), "bound": "tensor", "achieved": round(tf, 2), "peak": peak, "unit": "TFLOP/s",
            "frac": round(tf / peak, 4), "kernel": "out_proj_sm100_kernel",
            "traffic": OUT_PROJ_TRAFFIC.get((w.name, kernel_sources_hash(OUT_PROJ_SOURCES))),
            "algorithmic_bytes": 2 * (2 * M * K + K * C + 2 * M * C) + 2 * C,
            "cublas_reference": {"ms": round(ms_lib, 4), "tflops": round(fl / (ms_lib / 1e3) / 1e12, 2),
                                 "what": "torch.addmm + torch.mm (cuBLAS) on the same tensors"},
            "timing": "best of 2 alternating rounds of %d calls each" % steps}


def bench_cp_scatter(w, ins, steps, fl):
    """One rank's attention under P-way Ulysses context parallelism, emulated on
    this GPU: the rank's H/P heads over the whole sequence, written once to a
    plain [B, H/P, N, D] output and once scattered to the P sequence slices
    [B, H, N/P, D] (the epilogue doing the output all-to-all; the slices are
    local here, peer memory on a multi-GPU run). The two timings show what the
    scattered store costs in the kernel. No NVLink traffic is measured."""
    import masked_attention_jvp_b200 as caj
    P = next((p for p in (4, 2) if w.H % p == 0 and w.N % p == 0), None)
    if P is None:
        return None
    Hp, Ls = w.H // P, w.N // P
    mine = [x[:, :Hp].contiguous() for x in ins]
    dev = mine[0].device
    o = torch.empty(w.B, Hp, w.N, w.D, dtype=w.dtype, device=dev)
    to = torch.empty_like(o)
    lse = torch.empty(w.B, Hp, w.N, dtype=torch.float32, device=dev)
    tlse = torch.empty_like(lse)
    so = [torch.empty(w.B, w.H, Ls, w.D, dtype=w.dtype, device=dev) for _ in range(P)]
    sto = [torch.empty_like(t) for t in so]
    sl = [torch.empty(w.B, w.H, Ls, dtype=torch.float32, device=dev) for _ in range(P)]
    stl = [torch.empty_like(t) for t in sl]
    plain = lambda: caj.attn_fwd_jvp_out(*mine, w.mask, o, to, lse, tlse, scale=w.scale)
    scatter = lambda: caj.attn_fwd_jvp_scatter(*mine, w.mask, so, sto, sl, stl, head_base=0, scale=w.scale)
    res = {"ranks": P, "heads_per_rank": Hp, "slice_rows": Ls}
    # interleaved rounds, so that clock drift under the power cap hits both alike
    fns = {"plain": plain, "scatter": scatter}
    per_round = max(2, steps // 4)
    times = {k: [] for k in fns}
    for fn in fns.values():
        for _ in range(3):
            fn()
    torch.cuda.synchronize()
    for _ in range(4):
        for name, fn in fns.items():
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(per_round):
                fn()
            e1.record()
            torch.cuda.synchronize()
            times[name].append(e0.elapsed_time(e1) / per_round)
    for name, t in times.items():
        ms = statistics.median(t)
        res[f"ms_{name}"] = round(ms, 4)
        res[f"tflops_{name}"] = round(fl / P / (ms / 1e3) / 1e12, 2)
    res["scatter_over_plain"] = round(res["ms_scatter"] / res["ms_plain"], 4)
    return res


# ------------------------------------------------------- the other workloads
def bench_config(name, steps, warmup, peaks, with_cpu=True, cpu_target_s=5.0):
    """One of the other workloads, timed like the headline: `warmup` calls,
    then `steps` calls back to back with CUDA events, SM clocks sampled during
    the loop. The bf16 workloads run the tensor-core kernel and carry a
    roofline against the measured bf16 burst; the fp32 one runs the CUDA-core
    kernel (one small launch, bound by launch latency). The oracle is timed on
    a row sample of the same inputs beside it."""
    import masked_attention_jvp_b200 as caj
    w = WORKLOADS[name]
    dev = torch.device("cuda", torch.cuda.current_device())
    host = make_inputs(w, "cpu")
    ins = [t.to(dev) for t in host]
    shape = ins[0].shape
    o, to = torch.empty_like(ins[0]), torch.empty_like(ins[0])
    lse = torch.empty(shape[:3], dtype=torch.float32, device=dev)
    tlse = torch.empty_like(lse)
    fl = flops_of(w)

    def step():
        caj.attn_fwd_jvp_out(*ins, w.mask, o, to, lse, tlse, scale=w.scale)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    caj.device_status()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    with ClockSampler(dev.index) as clk:
        ev[0].record()
        for i in range(steps):
            step()
            ev[i + 1].record()
        torch.cuda.synchronize()
    caj.device_status()
    per = [ev[i].elapsed_time(ev[i + 1]) for i in range(steps)]
    ms = statistics.mean(per)
    tf = fl / (ms / 1e3) / 1e12
    res = {"workload": name, "B": w.B, "H": w.H, "N": w.N, "D": w.D, "mask": list(w.mask.as_tuple()),
           "dtype": "f32" if w.dtype == torch.float32 else "bf16",
           "flop_per_call": fl, "ms_mean": round(ms, 4), "ms_median": round(statistics.median(per), 4),
           "ms_min": round(min(per), 4), "tflops": round(tf, 3), "steps": steps, "warmup": warmup,
           "clocks": clk.summary(), "gpu_launches": steps}
    if w.dtype == torch.bfloat16:
        peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        res["kernel"] = "fwd_jvp_sm100_kernel<%d>" % w.D
        res["pct_of_dense_bf16_peak"] = round(100.0 * tf / DENSE_BF16_SPEC_TFLOPS, 2)
        res["roofline"] = {"bound": "tensor", "achieved": round(tf, 2), "peak": peak, "unit": "TFLOP/s",
                           "frac": round(tf / peak, 4), "peak_source": "measured bf16 burst (cuBLAS)"}
    else:
        res["kernel"] = "fwd_jvp_simt_f32_kernel<%d>" % w.D
        res["bound"] = "launch latency (one launch of %d CTAs; fp32 CUDA-core path for the 1e-5 tolerance)" % (
            w.B * w.H * ((w.N + 127) // 128))
    in_bytes = 6 * w.B * w.H * w.N * w.D * ins[0].element_size()
    res["l2"] = ("inputs larger than L2 (%.2f GB per step)" % (in_bytes / 1e9) if in_bytes > 126e6
                 else "inputs L2-resident (%.1f KB; a parity-size case timed for completeness)" % (in_bytes / 1e3))
    del ins, o, to, lse, tlse
    torch.cuda.empty_cache()
    if not with_cpu:
        return res
    ctf, dt, nrows, threads, desc = time_oracle(w, target_s=cpu_target_s, host_inputs=host)
    res["cpu_baseline"] = {"value": round(ctf, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                           "sample": desc, "seconds": round(dt, 2), "rows_per_s": round(nrows / dt, 1),
                           "extrapolated_full_call_s": round(fl / (ctf * 1e12), 2)}
    return res


# ------------------------------------------------------------------ GPU arm
def bench_e2e(args, w, host, fl_job, world, stream, dev, barrier):
    """Same metric through the public API from pinned host buffers: every step
    copies this rank's six inputs host->device and its four outputs
    device->host (attn_fwd_jvp on CPU tensors: the host-buffer entry point,
    which overlaps the copies with the kernels chunk by chunk). Timed over
    the same number of steps as the headline, clocks sampled meanwhile."""
    import masked_attention_jvp_b200 as caj
    pinned = [t.pin_memory() for t in host]
    h2d = sum(t.numel() * t.element_size() for t in pinned)
    n_rows = pinned[0].shape[0] * pinned[0].shape[1] * pinned[0].shape[2]
    d2h = 2 * n_rows * pinned[0].shape[3] * pinned[0].element_size() + 2 * n_rows * 4
    steps = args.steps
    have_work = pinned[0].numel() > 0
    if have_work:
        caj.attn_fwd_jvp(*pinned, w.mask, scale=w.scale)  # warm the host path once
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clk:
        e0.record(stream)
        for _ in range(steps):
            if have_work:
                caj.attn_fwd_jvp(*pinned, w.mask, scale=w.scale)
        e1.record(stream)
        torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    return {"value": round(strong_tflops(fl_job, steps, ms), 2), "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": round(ms / steps, 3), "clocks": clk.summary(),
            "api": "attn_fwd_jvp on pinned CPU tensors (caj_attn_fwd_jvp_host)"}


def rank_inputs(args, w, host, world, rank):
    """This rank's share of the workload's inputs (host tensors) and the
    problem it runs, by the split mode."""
    if world == 1 or args.split in ("replicas", "tiles"):
        return host, w  # tiles: every rank holds the whole inputs and runs its part of the query tiles
    if args.split == "heads":
        h0, h1 = split_heads(w.H, world, rank)
        return [t[:, h0:h1].contiguous() for t in host], w
    # ulysses: this rank's sequence shard of every head
    Ls = w.N // world
    return [t[:, :, rank * Ls:(rank + 1) * Ls].contiguous() for t in host], w


def bench_gpu(args, rank, world, local_rank):
    import masked_attention_jvp_b200 as caj

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = selected_workload(args)
    if args.split == "ulysses" and (w.H % world or w.N % world):
        raise SystemExit(f"--split ulysses needs heads ({w.H}) and tokens ({w.N}) divisible by {world} ranks")
    host_all = make_inputs(w, "cpu")
    if args.clean_tangent_zero:
        from masked_attention_jvp_b200.workloads import zero_clean_tangents
        zero_clean_tangents(w, *host_all[3:])
    host, _ = rank_inputs(args, w, host_all, world, rank)
    ins = [t.to(dev) for t in host]
    stream = torch.cuda.current_stream(dev)
    fl = flops_of(w)                                   # one copy of the whole problem
    fl_job = fl * (world if args.split == "replicas" else 1)
    have_work = ins[0].numel() > 0

    if args.split == "ulysses" and world > 1:
        from masked_attention_jvp_b200.ulysses import ulysses_attn_fwd_jvp

        def step():
            ulysses_attn_fwd_jvp(*ins, w.mask, scale=w.scale, clean_tangent_zero=args.clean_tangent_zero,
                                 fused_output=args.fused_output)
        launches_per_step = None  # NCCL kernels besides the library's
    else:
        o = torch.empty_like(ins[0])
        to = torch.empty_like(ins[0])
        lse = torch.empty(ins[0].shape[:3], dtype=torch.float32, device=dev)
        tlse = torch.empty_like(lse)

        part = (rank, world) if (args.split == "tiles" and world > 1) else None

        def step():
            if have_work:
                caj.attn_fwd_jvp_out(*ins, w.mask, o, to, lse, tlse, scale=w.scale, stream=stream,
                                     clean_tangent_zero=args.clean_tangent_zero, part=part)
        L = w.mask.n_frames * w.mask.tokens_per_frame
        launches_per_step = (2 if args.clean_tangent_zero and L >= 128 else 1) if have_work else 0

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    caj.device_status()

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    barrier()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    with ClockSampler(local_rank) as clk:
        ev[0].record(stream)
        for i in range(args.steps):
            step()
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
    barrier()
    caj.device_status()
    per = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    total_ms = max_over_ranks(ev[0].elapsed_time(ev[-1]), world, dev)
    ms_per_step = total_ms / args.steps
    value = strong_tflops(fl_job, args.steps, total_ms)

    # end to end through the public API with pinned host buffers
    e2e = None
    if not args.no_e2e and (world == 1 or args.split in ("heads", "replicas")):
        e2e = bench_e2e(args, w, host, fl_job, world, stream, dev, barrier)
    elif not args.no_e2e and args.split == "tiles":
        # host-resident inputs: a query-tile share would read every head's keys, so
        # each rank takes its share of the heads through the pipelined host call
        h0, h1 = split_heads(w.H, world, rank)
        share = [t[:, h0:h1].contiguous() for t in host]
        e2e = bench_e2e(args, w, share, fl_job, world, stream, dev, barrier)
        e2e["api"] += "; rank r its heads split_heads(H, world, r)"
    if rank != 0:
        return None
    peaks, src = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak_sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    kernel_ms = statistics.mean(per)
    rank0_flops = fl if (world == 1 or args.split == "replicas") else fl * (
        (split_heads(w.H, world, 0)[1] - split_heads(w.H, world, 0)[0]) / w.H if args.split == "heads" else 1.0 / world)
    # (tiles: the parts are balanced to within one query tile's work, so rank 0 does ~1/world)
    achieved = rank0_flops / (kernel_ms / 1e3) / 1e12
    clocks = clk.summary()
    parallelism = {"tiles": f"query tiles dealt over {world} GPUs by cost (every head)",
                   "heads": f"head split over {world} GPUs", "replicas": f"replica x{world}",
                   "ulysses": f"Ulysses context parallelism over {world} GPUs"
                              + (" (output all-to-all in the epilogue)" if args.fused_output else "")}[args.split]
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak" if args.split == "replicas" else "strong",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) q,k,v; N(0,0.5^2) tangents)",
        "config": workload_config(w, {"parallelism": parallelism if world > 1 else "single GPU"}),
        "pct_of_dense_bf16_peak": round(100.0 * value / world / DENSE_BF16_SPEC_TFLOPS, 2),
        "ms_per_step_min": round(min(per), 4), "ms_per_step_median": round(statistics.median(per), 4),
        "ms_per_step_each": [round(x, 3) for x in per],
        "clocks": clocks,
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps if launches_per_step is not None else None,
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4),
                     "frac_of_sustained": round(achieved / peak_sustained, 4),
                     "peak_sustained": peak_sustained,
                     "traffic": MEASURED_TRAFFIC.get((w.name, kernel_sources_hash())) if world == 1 else None,
                     "kernel_sources_sha256": kernel_sources_hash(),
                     "peak_source": f"{src} bf16 burst (cuBLAS)", "kernel": "fwd_jvp_sm100_kernel<128>"},
    }
    if world > 1:
        line["config"]["split"] = args.split
        if args.split == "heads":
            line["config"]["heads_per_rank"] = [b - a for a, b in (split_heads(w.H, world, r) for r in range(world))]
        if args.split == "ulysses" and args.fused_output:
            line["roofline"]["kernel"] = "fwd_jvp_sm100_kernel<128, scatter>"
    if args.clean_tangent_zero:
        line["roofline"]["traffic"] = None  # DRAM traffic was captured on dense inputs
        line["roofline"]["kernel"] = "fwd_jvp_sm100_kernel<128, noisy and clean tile kinds>"
        line["config"]["clean_tangent_zero"] = True
        line["products_tflop_per_step"] = round(ctz_product_flops(w) / 1e12, 3)
        line["roofline"]["achieved"] = round(ctz_product_flops(w) * rank0_flops / fl / (kernel_ms / 1e3) / 1e12, 2)
        line["roofline"]["frac"] = round(line["roofline"]["achieved"] / peak, 4)
        line["roofline"]["frac_of_sustained"] = round(line["roofline"]["achieved"] / peak_sustained, 4)
        line["roofline"]["note"] = "achieved counts only the products the kernel must do"
    if world > 1:
        return line   # the single-GPU legs below run at N = 1 only

    if not args.no_backward and not args.clean_tangent_zero:
        line["backward"] = bench_backward(w, ins, o, lse, args.steps, peaks)
        line["gpu_launches_backward"] = 3 * args.steps
    if not args.no_prologue:
        line["prologue"] = bench_prologue(w, dev, args.steps, peaks)
        line["gpu_launches_prologue"] = args.steps
    if not args.no_out_proj and not args.clean_tangent_zero:
        line["out_proj"] = bench_out_proj(w, dev, args.steps, peaks)
        line["gpu_launches_out_proj"] = 2 * (3 + args.steps)
    if w.mask.tf_layout and not args.clean_tangent_zero and not args.no_ctz:
        line["clean_tangent_zero"] = bench_ctz(w, ins, args.steps, fl)
    # last among the C2 legs: it heats the GPU, and the legs above keep their earlier conditions
    if not args.no_cp_scatter and not args.clean_tangent_zero:
        cp = bench_cp_scatter(w, ins, args.steps, fl)
        if cp is not None:
            line["cp_scatter"] = cp
            line["gpu_launches_cp_scatter"] = 2 * 4 * max(2, args.steps // 4)
    if not args.no_cpu_baseline:
        tf, dt, nrows, threads, desc = time_oracle(w, host_inputs=host_all)
        line["cpu_baseline"] = {"value": round(tf, 6), "unit": "TFLOP/s", "cores": threads,
                                "kind": "oracle", "sample": desc, "seconds": round(dt, 2),
                                "rows_per_s": round(nrows / dt, 1),
                                "extrapolated_full_call_s": round(fl / (tf * 1e12), 1),
                                "host": host_cpu()}
    if not args.no_configs and args.heads is None and not args.clean_tangent_zero:
        del ins, o, to, lse, tlse
        torch.cuda.empty_cache()
        line["configs"] = {}
        for name in WORKLOADS:
            if name == w.name:
                continue
            line["configs"][name] = bench_config(name, args.steps, args.warmup, peaks,
                                                 with_cpu=not args.no_cpu_baseline)
            torch.cuda.empty_cache()
        line["gpu_launches_configs"] = sum(c["gpu_launches"] for c in line["configs"].values())
    return line


def bench_reference(args, rank):
    """The oracle as it stands, on the host cores: each step a bounded row sample."""
    if rank != 0:
        return None
    import oracle
    from masked_attention_jvp_b200.workloads import sample_rows
    w = selected_workload(args)
    host = make_inputs(w, "cpu")
    threads = oracle.max_threads()
    per_head = 8
    rows_list = [sample_rows(w, per_head, seed_offset=200 + i) for i in range(args.warmup + args.steps)]
    for i in range(args.warmup):
        oracle.attn_fwd_jvp_rows(*host, w.mask, scale=w.scale, rows=rows_list[i])
    fl = 0
    t0 = time.perf_counter()
    for i in range(args.warmup, args.warmup + args.steps):
        oracle.attn_fwd_jvp_rows(*host, w.mask, scale=w.scale, rows=rows_list[i])
        fl += oracle_rows_flops(w, rows_list[i])
    dt = time.perf_counter() - t0
    value = fl / dt / 1e12
    desc = (f"per step {per_head} seeded query rows per head x {w.B * w.H} heads of {w.name}, "
            f"fp64 oracle, {threads} OpenMP threads")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * dt / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)", "config": workload_config(w),
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": desc, "host": host_cpu()},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def selected_workload(args):
    import dataclasses
    w = WORKLOADS[args.workload]
    if args.heads is not None:
        w = dataclasses.replace(w, name=f"{w.name}_h{args.heads}", H=args.heads)
    return w


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default=BENCH_WORKLOAD, choices=list(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--no-prologue", action="store_true", help="skip the prologue kernel's measurement")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward kernels' measurement")
    ap.add_argument("--no-out-proj", action="store_true", help="skip the output projection's measurement")
    ap.add_argument("--no-cp-scatter", action="store_true",
                    help="skip the context-parallel output-scatter measurement")
    ap.add_argument("--no-ctz", action="store_true",
                    help="skip the clean-tangent-zero sub-measurement (teacher-forcing workloads)")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip timing the other four workloads (the 'configs' key)")
    ap.add_argument("--split", default="tiles", choices=["tiles", "heads", "replicas", "ulysses"],
                    help="multi-GPU work split: the query tiles dealt over the ranks by cost (default, strong "
                         "scaling), the heads over the ranks, a copy per rank (weak scaling), or Ulysses sequence "
                         "shards with all-to-alls")
    ap.add_argument("--fused-output", action="store_true",
                    help="with --split ulysses: the output all-to-all in the attention epilogue")
    ap.add_argument("--heads", type=int, default=None,
                    help="override the workload's head count (small cases for ncu section captures)")
    ap.add_argument("--clean-tangent-zero", action="store_true",
                    help="TF-sCM inputs: zero clean tangents and let the kernel skip vanishing products "
                         "(value stays dense-equivalent 12*D per visible pair)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        line = bench_reference(args, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    try:
        line = bench_gpu(args, rank, world, local_rank)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
