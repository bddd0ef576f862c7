"""Benchmark of the HGRNBit block-stack forward on B200.

Workload (default): the 370M-shape stack, prefill forward, 24 HGRNBit blocks of hidden 1024 with
MLP gate_proj 1024->5632 and down_proj 2816->1024, vocabulary 32000 embedding, bf16 activations,
token ids uniform in [0, 32000) for batch 8 x sequence 2048 per GPU. Weights are random N(0, 0.02)
latent weights ternarised and 2-bit packed by the library. One step = one forward of the whole
stack (embedding gather + 24 blocks) over one batch; the tied head is not part of the prefill
step (it runs in the decode measurement, where generation needs it).

Prints one JSON line (rank 0). On one GPU the line also carries, as extra keys: the 2.7B-shape
greedy decode at batch 1 / 8 / 64 (every rank, as replicas), the 1.3B-shape prefill, the kernel
sweeps (BitLinear over three (K, N) shapes and five row counts; the HGRN scan at d 2048 up to
T 65536), the next-row kernels (HGRN2 recurrence, scan and BitLinear gradients) and two CPU
baselines (the oracle as written, and an fp32-BLAS restatement on every host core).

--impl reference times the CPU oracle on a bounded sample of the same workload instead.
--case NAME runs one kernel case a few times and prints its device time (profiler captures).
Multi-GPU runs are independent replicas (one batch per rank, no collective on the data path);
timing is the max over ranks.
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

METRIC = "HGRNBit block-stack tokens/s (prefill & decode, 1 B200); % HBM / INT8 roofline"
INT8_OVER_BF16 = 2.0  # nominal dense ratio: 4.5 POPS int8/fp8 vs 2.25 PFLOP/s bf16
# CUDA-core float32 FMA peak: 148 SMs x 128 FMA/clk x 2 flop x 1.965 GHz (the listed unit counts
# and the maximum SM clock)
FP32_FMA_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12

WORKLOADS = {
    "prefill-370M": dict(d=1024, inner=2816, layers=24, vocab=32000, batch=8, seq=2048),
    "prefill-1.3B": dict(d=2048, inner=5632, layers=24, vocab=32000, batch=16, seq=2048),
}
# DRAM traffic of one ternary_gemm_tc_kernel launch (dram__bytes_read.sum + dram__bytes_write.sum,
# averaged over the four GEMM launches of one block at this workload's per-launch shapes) from an ncu
# capture; valid only while the kernel source is the one captured (SHA-256 prefix), else null.
GEMM_TRAFFIC = {"prefill-370M": dict(bytes=79.0e6, algorithmic=115.2e6, sha256="d051d5284dbfdefd",
                                     profile="profiles/ternary_gemm_tc_kernel_prefill-370M_traffic.md")}
# Autoregressive decode of the 2.7B-shape stack: a 512-token prompt (prefill, untimed) then
# decode steps with the recurrent state carried per layer, at three batch sizes.
DECODE = dict(name="decode-2.7B", d=2560, inner=7040, layers=32, vocab=32000, prompt=512, batches=(1, 8, 64))
# Kernel sweeps (the pages' 1.3B layer shapes): BitLinear (K, N) x M, and the HGRN scan
SWEEP_BITLINEAR = dict(kn=((2048, 2048), (2048, 11264), (5632, 2048)), m=(1, 16, 256, 4096, 32768))
SWEEP_SCAN = dict(b=4, d=2048, t=(1024, 8192, 65536))


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="mmf", choices=["mmf", "reference"])
    ap.add_argument("--workload", default="prefill-370M", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the 1.3B prefill, sweeps and next-row kernels")
    ap.add_argument("--decode-steps", type=int, default=256)
    ap.add_argument("--case", default=None,
                    choices=["gemm", "scan", "block", "norm", "decode", "head", "hgrn2", "scan_bwd", "lin_bwd"],
                    help="run one kernel case and print its device time (for profiler captures)")
    ap.add_argument("--m", type=int, default=16384)
    ap.add_argument("--n", type=int, default=5632)
    ap.add_argument("--k", type=int, default=1024)
    ap.add_argument("--b", type=int, default=4)
    ap.add_argument("--t", type=int, default=8192)
    ap.add_argument("--d", type=int, default=1024)
    ap.add_argument("--inner", type=int, default=2816)
    ap.add_argument("--layers", type=int, default=4)
    ap.add_argument("--vocab", type=int, default=32000)
    ap.add_argument("--heads", type=int, default=8)
    ap.add_argument("--dtype", default="bf16", choices=["bf16", "f32"])
    ap.add_argument("--iters", type=int, default=5)
    ap.add_argument("--engine", default="auto", choices=["auto", "tensor", "simt"])
    ap.add_argument("--decode-path", default="auto", choices=["auto", "fused", "skinny", "block"])
    return ap.parse_args()


def load_peaks() -> dict:
    pp = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(pp):
        with open(pp) as fh:
            return json.load(fh)
    return {}


def int8_peak(peaks: dict) -> tuple[float, str]:
    """The int8 tensor peak for a kernel timed inside a step of milliseconds: the measured burst
    bf16 cuBLAS figure x the nominal int8/bf16 ratio (no int8 GEMM is measured on this machine)."""
    if peaks.get("bf16_tflops"):
        return (peaks["bf16_tflops"] * INT8_OVER_BF16,
                "of measured: bf16 burst cuBLAS x nominal int8/bf16 ratio 2 (the step lasts milliseconds)")
    return 1590.0 * INT8_OVER_BF16, "of fallback: 1.59 PFLOP/s bf16 burst x nominal ratio 2"


def bf16_peak(peaks: dict) -> tuple[float, str]:
    """The measured burst bf16 cuBLAS figure (for a kernel timed alone)."""
    if peaks.get("bf16_tflops"):
        return peaks["bf16_tflops"], "of measured: bf16 burst cuBLAS"
    return 1590.0, "of fallback: 1.59 PFLOP/s bf16 burst"


def hbm_peak(peaks: dict) -> tuple[float, str]:
    if peaks.get("hbm_gbs"):
        return peaks["hbm_gbs"], "of measured: STREAM-style copy"
    return 6650.0, "of fallback: 6.65 TB/s"


def gemm_traffic(workload: str):
    """Measured DRAM bytes per GEMM launch for this workload, or None when no capture matches the
    current kernel source."""
    import hashlib

    t = GEMM_TRAFFIC.get(workload)
    if t is None:
        return None
    src = os.path.join(ROOT, "ternary_weight_matmul_b200", "csrc", "gemm_tc.cuh")
    with open(src, "rb") as fh:
        if hashlib.sha256(fh.read()).hexdigest()[:16] != t["sha256"]:
            return None
    return t["bytes"]


def max_over_ranks(ms: float, device, world: int) -> float:
    """The slowest rank's time: replicas finish a step when the last one does."""
    import torch
    import torch.distributed as dist

    t = torch.tensor([ms], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def decode_entry(batch: int, ms_local: float, step_bytes: float, device, world: int, hbm_peak: float) -> dict:
    """One decode batch size across `world` replicas: each rank generates for its own `batch`
    sequences; the step time is the slowest rank's, the throughput the tokens of all replicas, and
    the bandwidth is per GPU (every replica streams its own copy of the weights)."""
    ms = max_over_ranks(ms_local, device, world)
    gbs = step_bytes / (ms / 1e3) / 1e9
    return {"value": batch * world / (ms / 1e3), "ms_per_step": ms, "replicas": world,
            "bytes_per_step": step_bytes, "GB/s": gbs, "frac_hbm": gbs / hbm_peak}


def replicas_throughput(tokens_per_rank: int, world: int, ms_max: float) -> float:
    """Whole-job tokens/s of `world` independent replicas, each processing its own batch."""
    return tokens_per_rank * world / (ms_max / 1e3)


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


# ---------------------------------------------------------------------------------------------
# CPU baselines: the oracle (reference arm and cpu_baseline) and an fp32-BLAS restatement
# ---------------------------------------------------------------------------------------------
_ORACLE_LAYER = {}


def oracle_sample_tokens_per_s(wl: dict, tokens: int, seed: int = 0) -> tuple[float, str, float]:
    """Times the oracle's block forward for one layer of the workload on one sequence of
    `tokens` tokens and extrapolates linearly to the whole stack (the work is linear in tokens
    and layers). Returns (tokens/s of the full stack, sample description, seconds). The layer's
    weights are drawn and ternarised once, outside the timing."""
    import numpy as np

    import oracle as O
    import synth

    key = (wl["d"], wl["inner"])
    if key not in _ORACLE_LAYER:
        shape = synth.BlockShape("bench", wl["d"], wl["inner"], 1)
        _ORACLE_LAYER[key] = O.quantize_block(synth.block_params(0, shape))
    qp = _ORACLE_LAYER[key]
    table = synth.embedding(seed + 1, 1000, wl["d"])
    ids = synth.token_ids(seed + 2, (1, tokens), vocab=1000)
    x = O.embed(ids, table)
    t0 = time.perf_counter()
    O.block_forward(x.astype(np.float64), qp)
    dt = time.perf_counter() - t0
    per_token_stack = dt / tokens * wl["layers"]
    desc = (f"oracle (numpy float64/int64) block forward of 1 of {wl['layers']} layers on 1 sequence of "
            f"{tokens} tokens, extrapolated linearly to {wl['layers']} layers")
    return 1.0 / per_token_stack, desc, dt


def oracle_threads() -> int:
    for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        if os.environ.get(var):
            try:
                return int(os.environ[var])
            except ValueError:
                pass
    return 1  # the integer product and the scan loop run on one core; BLAS is not used


def cpu_fast_tokens_per_s(wl: dict, tokens: int, seed: int = 0) -> tuple[float, str, float, int]:
    """A fast CPU baseline (timing only; never called by the library): the block forward
    restated with torch CPU tensors in float32 on every host core. The integer product runs as an
    fp32 BLAS product of the int8 codes and the ternary codes, which is exact: every partial sum
    is an integer of magnitude <= 127 * K < 2^24. The recurrence is a loop over time, vectorised
    over the channels. One layer on one sequence of `tokens` tokens, extrapolated linearly to the
    stack. Returns (tokens/s, description, seconds, threads)."""
    import torch

    threads = os.cpu_count() or 1
    torch.set_num_threads(threads)
    g = torch.Generator().manual_seed(seed)
    d, inner, eps = wl["d"], wl["inner"], 1e-8
    shapes = {"i": (d, d), "f": (d, d), "g": (d, d), "o": (d, d), "gate": (2 * inner, d), "down": (d, inner)}
    lay = {}
    for p, (n, k) in shapes.items():
        w = torch.randn(n, k, generator=g) * 0.02
        s = w.abs().mean().clamp_min(1e-5)
        lay[p] = ((w / s).round().clamp(-1, 1).t().contiguous(), float(s))  # [K, N] float32 codes
    x = torch.randn(1, tokens, d, generator=g)

    def bitlinear(v, tt, s):
        r = v * torch.rsqrt((v * v).mean(-1, keepdim=True) + eps)
        a = r.abs().amax(-1, keepdim=True).clamp_min(1e-5)
        q = torch.round(r * (127.0 / a)).clamp(-127, 127)
        return (q @ tt) * (a / 127.0) * s

    def block(v):
        zi, zf, gg = (bitlinear(v, *lay[p]) for p in ("i", "f", "g"))
        f = torch.sigmoid(zf)
        i = torch.nn.functional.silu(zi) * (1 - f)
        h = torch.empty_like(i)
        prev = torch.zeros(v.shape[0], d)
        for t in range(v.shape[1]):
            prev = f[:, t] * prev + i[:, t]
            h[:, t] = prev
        u = h * torch.rsqrt((h * h).mean(-1, keepdim=True) + eps) * torch.nn.functional.silu(gg)
        x1 = v + bitlinear(u, *lay["o"])
        gu = bitlinear(x1, *lay["gate"])
        vv = torch.nn.functional.silu(gu[..., :inner]) * gu[..., inner:]
        return x1 + bitlinear(vv, *lay["down"])

    block(x[:, :64])  # warm-up (thread pool, BLAS)
    t0 = time.perf_counter()
    block(x)
    dt = time.perf_counter() - t0
    desc = (f"torch CPU float32 restatement (fp32 BLAS on the int8 x ternary codes, exact; recurrence "
            f"vectorised over d) of 1 of {wl['layers']} layers on 1 sequence of {tokens} tokens, "
            f"extrapolated linearly to {wl['layers']} layers")
    return tokens / (dt * wl["layers"]), desc, dt, threads


def run_reference(args, wl):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    tokens = 48  # one step = one bounded sample (about a second of CPU work)
    for _ in range(args.warmup):
        oracle_sample_tokens_per_s(wl, tokens)
    times = []
    t_all = time.perf_counter()
    for i in range(args.steps):
        _, desc, dt = oracle_sample_tokens_per_s(wl, tokens, seed=i)
        times.append(dt)
    wall = time.perf_counter() - t_all
    per_step_stack = statistics.mean(times) * wl["layers"]  # seconds per `tokens` tokens, whole stack
    value = tokens / per_step_stack
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step_stack * 1e3,
        "ms_per_step_kind": (f"extrapolated: each step times 1 of {wl['layers']} layers on {tokens} tokens "
                             f"and scales by {wl['layers']}; the stack itself is never run"),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64 / int64 (oracle)", "data": "synthetic",
        "config": {"workload": args.workload, **{k: wl[k] for k in ("d", "inner", "layers", "vocab")},
                   "sample_tokens_per_step": tokens},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle_threads(), "kind": "oracle",
                         "sample": desc, "host_cpus": os.cpu_count()},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": wall,
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------------------------
# clocks sampling
# ---------------------------------------------------------------------------------------------
class Clocks:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(prefix="mmf_clocks_", suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict | None:
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as fh:
            for line in fh:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------------------------
def build_model(wl, device, seed=1234):
    """Random N(0, 0.02) latent weights drawn on the device with a seeded generator, packed by the
    library; norm gains are ones (the usual init). The embedding table is N(0, 0.02) in bf16."""
    import torch

    import ternary_weight_matmul_b200 as mmf

    g = torch.Generator(device=device)
    g.manual_seed(seed)
    d, inner = wl["d"], wl["inner"]
    shapes = {"i": (d, d), "f": (d, d), "g": (d, d), "o": (d, d), "gate": (2 * inner, d), "down": (d, inner)}
    blocks = []
    for _ in range(wl["layers"]):
        packed, norms = {}, {}
        for p, (n, k) in shapes.items():
            w = torch.randn(n, k, generator=g, device=device, dtype=torch.float32).mul_(0.02)
            packed[p] = mmf.pack_ternary(w)
            del w
            norms[f"nw_{p}"] = torch.ones(k, device=device, dtype=torch.float32)
        norms["gnorm_w"] = torch.ones(d, device=device, dtype=torch.float32)
        blocks.append(mmf.Block(d, inner, packed, norms))
    table = (torch.randn(wl["vocab"], d, generator=g, device=device) * 0.02).to(torch.bfloat16)
    return blocks, table


def kernel_classes(mmf) -> dict:
    """Per kernel class: launches, device ms and algorithmic work recorded since the last read."""
    out = {}
    for cls in ("gemm_tc", "gemm_simt", "norm_quant", "scan", "other"):
        n, kms, work = mmf.timing_read(cls)
        out[cls] = {"launches": n, "ms": kms, "work": work}
    return out


def hbm_breakdown(kern: dict, total_ms: float, hbm: float) -> dict:
    out = {}
    for cls in ("norm_quant", "scan", "gemm_simt", "other"):
        k = kern[cls]
        if k["launches"]:
            gbs = k["work"] / (k["ms"] / 1e3) / 1e9
            out[cls] = {"launches": k["launches"], "ms_total": k["ms"], "GB/s": gbs, "frac_hbm": gbs / hbm,
                        "share_of_step": k["ms"] / total_ms}
    return out


def run_decode(args, device, hbm, world=1):
    """Greedy autoregressive decode throughput of the 2.7B-shape stack for each batch size: prompt
    prefill through mmf_stack_fwd (untimed; gives every layer's recurrent state and, through the
    final norm and the tied head, the first generated token), then `--decode-steps` generated
    tokens, each step = embedding gather of the current ids + mmf_decode_step + final RMSNorm,
    tied head and argmax (mmf_lm_head_argmax writes the next ids in place), replayed from a CUDA
    graph (captured after warm-up) and timed with CUDA events on the replay stream. HBM roofline:
    every step streams all packed weights and the bf16 head table (once per pass of the head: one
    row on the CUDA cores, up to 128 rows on the tensor cores). Then a few steps run eagerly with
    the library's per-launch events on, which attribute the step time to the kernel classes. With
    several ranks every rank is a replica generating for its own sequences; the ranks meet at a
    barrier before each timed region and the step time is the slowest rank's."""
    import torch
    import torch.distributed as dist

    import ternary_weight_matmul_b200 as mmf

    dw = DECODE
    blocks, table = build_model(dw, device, seed=2718)
    weight_bytes = 0
    for blk in blocks:
        for p in blk.packed.values():
            weight_bytes += p.codes.numel() * 4 + 4
        weight_bytes += sum(t.numel() * 4 for t in blk.norms.values())
    fnorm = torch.ones(dw["d"], dtype=torch.float32, device=device)  # final RMSNorm gain
    head_bytes = table.numel() * table.element_size()
    out = {"workload": dw["name"], "layers": dw["layers"], "hidden": dw["d"], "inner": dw["inner"],
           "prompt": dw["prompt"], "steps": args.decode_steps, "unit": "tokens/s",
           "generation": "greedy (final RMSNorm + tied head + argmax on the GPU, ids fed back)",
           "bytes_per_step_weights": weight_bytes, "bytes_head_table": head_bytes, "batches": {}}
    for B in dw["batches"]:
        g = torch.Generator(device="cpu")
        g.manual_seed(99 + B)
        prompt = torch.randint(0, dw["vocab"], (B, dw["prompt"]), generator=g, dtype=torch.int32).to(device)
        yp, state = mmf.stack_fwd(blocks, prompt, table, want_state=True)
        x = torch.empty(B, dw["d"], dtype=torch.bfloat16, device=device)
        y = torch.empty_like(x)
        cur = torch.empty(B, dtype=torch.int32, device=device)
        mmf.lm_head_argmax(yp[:, -1, :].contiguous(), fnorm, table, ids_out=cur)  # first generated token
        s = torch.cuda.Stream(device)

        def step():
            xx = mmf.embed_gather(cur, table)
            x.copy_(xx)
            mmf.decode_step(blocks, x, state, out=y)
            mmf.lm_head_argmax(y, fnorm, table, ids_out=cur)

        with torch.cuda.stream(s):
            for i in range(3):
                step()
        torch.cuda.synchronize(device)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            step()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(s):
            for i in range(3):
                graph.replay()
            torch.cuda.synchronize(device)
            if world > 1:
                dist.barrier()
            ev0.record(s)
            for i in range(args.decode_steps):
                graph.replay()
            ev1.record(s)
        torch.cuda.synchronize(device)
        st = mmf.sync_status(device)
        if st != 0:
            raise RuntimeError(f"device status {st} in decode")
        ms = ev0.elapsed_time(ev1) / args.decode_steps
        step_bytes = weight_bytes + head_bytes * ((B + 127) // 128)
        ids_end = cur.cpu()
        assert int(ids_end.min()) >= 0 and int(ids_end.max()) < dw["vocab"]
        entry = decode_entry(B, ms, step_bytes, device, world, hbm)
        # per-class attribution from a few eager steps with the library's launch events
        kernel_classes(mmf)  # clear
        n_eager = 4
        with torch.cuda.stream(s):
            mmf.timing_enable(True)
            for i in range(n_eager):
                step()
            torch.cuda.synchronize(device)
            mmf.timing_enable(False)
        kern = kernel_classes(mmf)
        cls_ms = {c: v["ms"] / n_eager for c, v in kern.items() if v["launches"]}
        dom = max(cls_ms, key=cls_ms.get)
        path = {mmf.MMF_DECODE_FUSED: "fused", mmf.MMF_DECODE_SKINNY: "skinny",
                mmf.MMF_DECODE_BLOCK: "block"}.get(mmf.decode_path(B, dw["d"], dw["inner"]), "?")
        names = {"gemm_tc": "ternary_gemm_skinny_kernel" if path == "skinny" else "ternary_gemm_tc_kernel",
                 "gemm_simt": "dec_proj_kernel" if path == "fused" else "simt_gemm_kernel",
                 "norm_quant": "row_stage_kernel" if path == "skinny" else "norm_quant_vec_kernel",
                 "scan": "scan kernels", "other": "head / gather kernels"}
        gemm_ms = sum(cls_ms.get(c, 0.0) for c in ("gemm_tc", "gemm_simt"))
        gemm_gbs = weight_bytes / (gemm_ms / 1e3) / 1e9 if gemm_ms > 0 else None
        entry["path"] = path
        entry["roofline"] = {
            "bound": "hbm", "dominant": names[dom], "dominant_ms_per_step": cls_ms[dom],
            "launches_per_step": {c: kern[c]["launches"] / n_eager for c in kern if kern[c]["launches"]},
            "ms_per_step_by_class": cls_ms,
            "weight_products_ms_per_step": gemm_ms,
            "weight_products_GB/s": gemm_gbs, "weight_products_frac_hbm": gemm_gbs / hbm if gemm_gbs else None,
            "note": "class times from eager steps with per-launch events (launch gaps excluded); "
                    "the step time above is the graph replay"}
        out["batches"][str(B)] = entry
        del graph
    del blocks, table
    torch.cuda.empty_cache()
    return out


def time_prefill(wl, device, steps, warmup, flush, clocks=None):
    """Device time of the block-stack prefill step over one batch (seeded ids), L2 flushed between
    steps; returns (ms per step list, kernel classes, launches, ids_host, blocks, table, y)."""
    import torch

    import ternary_weight_matmul_b200 as mmf

    rank = dist_env()[0]
    blocks, table = build_model(wl, device)
    B, T, d = wl["batch"], wl["seq"], wl["d"]
    g = torch.Generator(device="cpu")
    g.manual_seed(4321 + rank)
    ids_host = torch.randint(0, wl["vocab"], (B, T), generator=g, dtype=torch.int32).pin_memory()
    ids = ids_host.to(device)
    y = torch.empty(B, T, d, dtype=torch.bfloat16, device=device)

    def step():
        mmf.stack_fwd(blocks, ids, table, out=y)

    for _ in range(max(warmup, 3)):
        flush.zero_()
        step()
    st = mmf.sync_status(device)
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up")
    stream = torch.cuda.current_stream(device)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    return blocks, table, ids_host, y, step, stream, starts, ends


def gemm_roofline(kern: dict, total_ms: float, peak: float, peak_src: str, workload: str | None) -> dict:
    tc = kern["gemm_tc"]
    achieved = (tc["work"] / (tc["ms"] / 1e3) / 1e12) if tc["ms"] > 0 else 0.0
    r = {"bound": "tensor", "kernel": "ternary_gemm_tc_kernel", "achieved": achieved, "peak": peak,
         "unit": "TOPS (int8)", "frac": achieved / peak, "peak_source": peak_src,
         "launches": tc["launches"], "avg_launch_us": tc["ms"] / max(tc["launches"], 1) * 1e3,
         "share_of_step": tc["ms"] / total_ms}
    if workload is not None:
        r.update({"traffic": gemm_traffic(workload),
                  "traffic_source": GEMM_TRAFFIC.get(workload, {}).get("profile"),
                  "algorithmic_bytes_per_launch": GEMM_TRAFFIC.get(workload, {}).get("algorithmic")})
    return r


def run_prefill_extra(wl_name, device, flush, peaks) -> dict:
    """A second prefill workload (the 1.3B shape), device time only, as an extra key."""
    import torch

    import ternary_weight_matmul_b200 as mmf

    wl = WORKLOADS[wl_name]
    blocks, table, ids_host, y, step, stream, starts, ends = time_prefill(wl, device, 5, 3, flush)

    def timed(instrumented):
        mmf.timing_enable(instrumented)
        for i in range(5):
            flush.zero_()
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        torch.cuda.synchronize(device)
        mmf.timing_enable(False)
        if mmf.sync_status(device) != 0:
            raise RuntimeError(f"device status after {wl_name}")
        return statistics.mean(s.elapsed_time(e) for s, e in zip(starts, ends))

    ms = timed(False)          # the step time, no per-launch events
    ms_attr = timed(True)      # the same steps again for the kernel classes
    kern = kernel_classes(mmf)
    peak, src = int8_peak(peaks)
    hbm, _ = hbm_peak(peaks)
    tokens = wl["batch"] * wl["seq"]
    out = {"workload": wl_name, "value": tokens / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
           "ms_per_step_with_launch_events": ms_attr,
           "steps": 5, "config": wl, "roofline": gemm_roofline(kern, ms_attr * 5, peak, src, None),
           "hbm_kernels": hbm_breakdown(kern, ms_attr * 5, hbm)}
    del blocks, table, y
    torch.cuda.empty_cache()
    return out


def run_sweeps(device, flush, peaks) -> dict:
    """Kernel sweeps: each BitLinear call (norm-quant + product) and each scan timed alone with CUDA
    events, L2 flushed before every repetition; the median of the repetitions is reported against
    its roofline (HBM bytes below the ridge, int8 ops above it)."""
    import torch

    import ternary_weight_matmul_b200 as mmf

    peak, _ = int8_peak(peaks)
    hbm, _ = hbm_peak(peaks)
    g = torch.Generator(device=device)
    g.manual_seed(77)
    stream = torch.cuda.current_stream(device)
    reps = 8

    def median_ms(fn, classes=False):
        # the call times carry no per-launch events; with `classes`, the same number of calls
        # again with the library's launch events gives the product kernel's own time
        times, kern_total = [], None
        for r in range(reps + 2):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize(device)
            if r >= 2:
                times.append(a.elapsed_time(b))
        if classes:
            kernel_classes(mmf)  # clear
            for _ in range(reps):
                flush.zero_()
                mmf.timing_enable(True)
                fn()
                torch.cuda.synchronize(device)
                mmf.timing_enable(False)
            kern_total = kernel_classes(mmf)
        return statistics.median(times), kern_total

    bl = []
    for k, n in SWEEP_BITLINEAR["kn"]:
        w = mmf.pack_ternary(torch.randn(n, k, generator=g, device=device) * 0.02)
        for m in SWEEP_BITLINEAR["m"]:
            x = torch.randn(m, k, generator=g, device=device).to(torch.bfloat16)
            yb = torch.empty(m, n, dtype=torch.bfloat16, device=device)
            ms, kern = median_ms(lambda: mmf.bitlinear_fwd(x, None, w, y_dtype=torch.bfloat16), classes=True)
            ops = 2.0 * m * n * k
            byts = n * (k // 4) + 2.0 * m * k + 2.0 * m * n
            e = {"K": k, "N": n, "M": m, "call_ms": ms, "call_TOPS": ops / (ms / 1e3) / 1e12,
                 "call_GB/s": byts / (ms / 1e3) / 1e9}
            gk = "gemm_tc" if kern["gemm_tc"]["launches"] else "gemm_simt"
            gms = kern[gk]["ms"] / reps
            e["product_kernel"] = "ternary_gemm_tc_kernel" if gk == "gemm_tc" else "simt_gemm_kernel"
            e["product_ms"] = gms
            if m <= 16:
                gbs = (n * (k // 4) + m * k + 2.0 * m * n) / (gms / 1e3) / 1e9
                e.update({"bound": "hbm", "product_GB/s": gbs, "frac": gbs / hbm})
            else:
                tops = ops / (gms / 1e3) / 1e12
                e.update({"bound": "tensor", "product_TOPS": tops, "frac": tops / peak})
            bl.append(e)
            del x, yb
        del w
    torch.cuda.empty_cache()
    sc = []
    b, d = SWEEP_SCAN["b"], SWEEP_SCAN["d"]
    for t in SWEEP_SCAN["t"]:
        zf = torch.randn(b, t, d, generator=g, device=device).add_(4.0)
        zi = torch.randn(b, t, d, generator=g, device=device)
        ms, _ = median_ms(lambda: mmf.hgrn_scan(zf, zi, None, h_dtype=torch.float32))
        byts = 12.0 * b * t * d
        gbs = byts / (ms / 1e3) / 1e9
        sc.append({"B": b, "T": t, "d": d, "dtype": "f32 in / f32 out", "ms": ms, "GB/s": gbs, "frac_hbm": gbs / hbm,
                   "bytes": byts})
        del zf, zi
    torch.cuda.empty_cache()
    return {"bitlinear": bl, "scan": sc, "reps": reps, "l2": "flushed before every repetition",
            "activations": "N(0,1) bf16 (BitLinear); scan gates zf ~ N(4,1), zi ~ N(0,1) float32"}


def run_next_rows(device, flush, peaks) -> dict:
    """The next-row kernels timed alone (median of a few calls, L2 flushed before each): the HGRN2
    recurrence (step by step on the CUDA cores), the scan gradients and the BitLinear gradients
    (straight-through estimator; dr and dW on the bf16 tensor cores)."""
    import torch

    import ternary_weight_matmul_b200 as mmf

    hbm, _ = hbm_peak(peaks)
    g = torch.Generator(device=device)
    g.manual_seed(88)
    stream = torch.cuda.current_stream(device)

    def median_ms(fn, reps=5):
        ts = []
        for r in range(reps + 1):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize(device)
            if r:
                ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    out = {}
    # HGRN2: 8 sequences x 2048 steps, 8 heads of dk = dv = 128 (hidden 1024), bf16
    B, T, H, dk = 8, 2048, 8, 128
    q = torch.randn(B, T, H, dk, generator=g, device=device).to(torch.bfloat16)
    f = torch.sigmoid(torch.randn(B, T, H, dk, generator=g, device=device) + 2).to(torch.bfloat16)
    i = torch.randn(B, T, H, dk, generator=g, device=device).to(torch.bfloat16)
    ms = median_ms(lambda: mmf.hgrn2_recurrence(q, f, i))
    flops = 4.0 * B * T * H * dk * dk   # per (step, head): dk x dv decay-and-add FMAs + the dk x dv readout
    byts = 2.0 * B * T * H * (3 * dk)   # q, f, i in and o out in bf16 (q, f shared across columns)
    out["hgrn2_recurrence"] = {"shape": f"B {B} T {T} heads {H} dk {dk} dv {dk} bf16", "ms": ms,
                               "TFLOP/s": flops / (ms / 1e3) / 1e12,
                               "frac_fp32_fma_peak": flops / (ms / 1e3) / 1e12 / FP32_FMA_TFLOPS,
                               "GB/s": byts / (ms / 1e3) / 1e9, "bound": "alu",
                               "peak_source": "CUDA-core fp32 FMA peak from unit counts x 1.965 GHz"}
    del q, f, i
    # scan backward: 8 x 2048 x 1024 bf16 (the 370M prefill shape)
    B, T, d = 8, 2048, 1024
    zf = torch.randn(B, T, d, generator=g, device=device).add_(2).to(torch.bfloat16)
    zi = torch.randn(B, T, d, generator=g, device=device).to(torch.bfloat16)
    h, _ = mmf.hgrn_scan(zf, zi, None, h_dtype=torch.bfloat16)
    dh = torch.randn(B, T, d, generator=g, device=device).to(torch.bfloat16)
    ms = median_ms(lambda: mmf.hgrn_scan_backward(zf, zi, h, dh))
    byts = 6.0 * 2 * B * T * d
    out["hgrn_scan_backward"] = {"shape": f"B {B} T {T} d {d} bf16", "ms": ms, "GB/s": byts / (ms / 1e3) / 1e9,
                                 "frac_hbm": byts / (ms / 1e3) / 1e9 / hbm, "bound": "hbm"}
    del zf, zi, h, dh
    # BitLinear backward, bf16 activations and gradients: 4096 rows with K = N = 1024, and the
    # 370M prefill's gate_proj (16384 rows, K 1024, N 2816). The whole call (operand layout, the
    # two tensor-core products, rho, the gain's gradient, dx) against the bf16 tensor peak for
    # dr + dW's algorithmic 4 m n k flops (the hi / lo pairs issue twice that on the MMA)
    bpk, bsrc = bf16_peak(peaks)
    for key, (m, k, n) in (("bitlinear_backward", (4096, 1024, 1024)),
                           ("bitlinear_backward_370M_gate", (16384, 1024, 2816))):
        w = mmf.pack_ternary(torch.randn(n, k, generator=g, device=device) * 0.02)
        x = torch.randn(m, k, generator=g, device=device).to(torch.bfloat16)
        nw = torch.ones(k, device=device)
        _, qq, deq, _ = mmf.bitlinear_fwd(x, nw, w, y_dtype=torch.float32, debug=True)
        dy = torch.randn(m, n, generator=g, device=device).to(torch.bfloat16)
        ms = median_ms(lambda: mmf.bitlinear_backward(x, nw, w, qq, deq, dy))
        flops = 2 * 2.0 * m * n * k   # dr and dW
        out[key] = {"shape": f"M {m} K {k} N {n} bf16", "ms": ms, "TFLOP/s": flops / (ms / 1e3) / 1e12,
                    "frac_bf16_peak": flops / (ms / 1e3) / 1e12 / bpk, "bound": "tensor", "peak_source": bsrc}
        del w, x, qq, deq, dy
    if mmf.sync_status(device) != 0:
        raise RuntimeError("device status after the next-row kernels")
    return out


def guarded(fn, *args):
    """One extra measurement of the JSON line: a failure there is reported in its entry (and its
    traceback on stderr) instead of losing the headline line. Used on one GPU only, where no other
    rank waits in a collective."""
    try:
        return fn(*args)
    except Exception as e:  # noqa: BLE001 -- any failure of an extra is reported, not raised
        import traceback

        traceback.print_exc(file=sys.stderr)
        return {"error": f"{type(e).__name__}: {e}"}


def run_gpu(args, wl):
    import torch
    import torch.distributed as dist

    import ternary_weight_matmul_b200 as mmf

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", device_id=device, timeout=__import__("datetime").timedelta(seconds=300))

    mmf.lib()
    peaks = load_peaks()
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device=device)
    blocks, table, ids_host, y, step, stream, starts, ends = time_prefill(wl, device, args.steps, args.warmup, flush)
    B, T, d = wl["batch"], wl["seq"], wl["d"]

    # ---------------- timed region (device time, events on the launching stream)
    clocks = Clocks(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(device)
    clocks.start()
    time.sleep(0.3)
    launches0 = mmf.launch_count()
    for i in range(args.steps):
        flush.zero_()  # write a buffer larger than L2 between steps (not timed)
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize(device)
    launches = mmf.launch_count() - launches0
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    st = mmf.sync_status(device)
    if st != 0:
        raise RuntimeError(f"device status {st} in the timed region")
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    ms = sum(step_ms) / len(step_ms)
    ms_max = max_over_ranks(ms, device, world)
    value = replicas_throughput(B * T, world, ms_max)
    gpu_launches = int(launches)  # our kernels launched in the timed region (counted by the library)

    # ---------------- attribution: the same K steps again with the library's per-launch events
    # on the launching stream (kernel classes, the roofline's per-launch durations). Kept out of
    # the headline steps above: the events between launches cost about 2-4% of a step.
    if world > 1:
        dist.barrier()
    mmf.timing_enable(True)
    a_s = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    a_e = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for i in range(args.steps):
        flush.zero_()
        a_s[i].record(stream)
        step()
        a_e[i].record(stream)
    torch.cuda.synchronize(device)
    mmf.timing_enable(False)
    kern = kernel_classes(mmf)
    ms_attr = sum(s.elapsed_time(e) for s, e in zip(a_s, a_e)) / args.steps

    # ---------------- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        # A serving loop: every step copies its ids in from pinned host memory, runs the stack
        # through the public API and copies its hidden states back to pinned host memory; the
        # copy back of step i runs on a copy stream while step i + 1 computes (two output
        # buffers, each reused only after its copy has finished). One timed region from the
        # first step's copy in to the last step's copy back, the L2 flushes between steps inside.
        y_bufs = [y, torch.empty_like(y)]
        y_host = [torch.empty(B, T, d, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        copy_s = torch.cuda.Stream(device)
        computed = [torch.cuda.Event() for _ in range(args.steps)]
        copied = [torch.cuda.Event() for _ in range(args.steps)]
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(device)
        e0.record(stream)
        for i in range(args.steps):
            if i >= 2:
                stream.wait_event(copied[i - 2])  # this output buffer's copy back has finished
            flush.zero_()
            ids_dev = ids_host.to(device, non_blocking=True)
            yy, _ = mmf.stack_fwd(blocks, ids_dev, table, out=y_bufs[i % 2])
            computed[i].record(stream)
            copy_s.wait_event(computed[i])
            with torch.cuda.stream(copy_s):
                y_host[i % 2].copy_(yy, non_blocking=True)
            copied[i].record(copy_s)
        stream.wait_event(copied[args.steps - 1])
        e1.record(stream)
        torch.cuda.synchronize(device)
        if mmf.sync_status(device) != 0:
            raise RuntimeError("device status in the end-to-end steps")
        e_ms = e0.elapsed_time(e1) / args.steps
        e2e = {"value": replicas_throughput(B * T, world, max_over_ranks(e_ms, device, world)), "unit": "tokens/s",
               "h2d_bytes_per_step": ids_host.numel() * 4, "d2h_bytes_per_step": y_host[0].numel() * 2,
               "ms_per_step": e_ms,
               "pipeline": "copy back of step i overlaps step i+1 (copy stream, two output buffers); "
                           "one timed region, L2 flushes between steps included"}
    del blocks, table, y
    torch.cuda.empty_cache()

    hbm, hbm_src = hbm_peak(peaks)
    decode = None
    if not args.no_decode:  # every rank: decode replicas, timed as the slowest rank
        decode = run_decode(args, device, hbm, world) if world > 1 else guarded(run_decode, args, device, hbm, world)

    extra = {}
    if world == 1 and not args.no_extra:
        extra["prefill-1.3B"] = guarded(run_prefill_extra, "prefill-1.3B", device, flush, peaks)
        extra["sweeps"] = guarded(run_sweeps, device, flush, peaks)
        extra["next_rows"] = guarded(run_next_rows, device, flush, peaks)

    line = None
    if rank == 0:
        peak, peak_src = int8_peak(peaks)
        roofline = gemm_roofline(kern, ms_attr * args.steps, peak, peak_src, args.workload)
        roofline["attribution"] = (f"per-launch events over a second pass of the {args.steps} timed steps "
                                   f"({ms_attr:.3f} ms per step with the events, {ms:.3f} without)")
        hbm_kernels = hbm_breakdown(kern, ms_attr * args.steps, hbm)
        cpu = cpu_fast = None
        if not args.no_cpu_baseline and world == 1:
            v, desc, dt = oracle_sample_tokens_per_s(wl, 1024)
            cpu = {"value": v, "unit": "tokens/s", "cores": oracle_threads(), "kind": "oracle",
                   "sample": desc + f" ({dt:.1f} s)", "host_cpus": os.cpu_count()}
            v, desc, dt, thr = cpu_fast_tokens_per_s(wl, 2048)
            cpu_fast = {"value": v, "unit": "tokens/s", "cores": thr, "kind": "fp32 BLAS restatement (exact)",
                        "sample": desc + f" ({dt:.2f} s)", "host_cpus": os.cpu_count()}
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "s8 x ternary -> s32 GEMM; bf16 activations, f32 reductions",
            "data": "synthetic (seeded random N(0,0.02) ternarised weights, uniform token ids)",
            "config": {"workload": args.workload, "model": "HGRNBit stack (random init)",
                       "global_batch": B * world, "seq_len": T, "hidden": d, "inner": wl["inner"],
                       "layers": wl["layers"], "vocab": wl["vocab"], "parallelism": f"replicas x{world}",
                       "head": "excluded (block stack only; the tied head runs in the decode measurement)",
                       "l2": "flushed between steps (write of a 2x-L2 buffer, untimed)"},
            "roofline": roofline, "hbm_kernels": hbm_kernels, "hbm_peak_gbs": hbm, "hbm_peak_source": hbm_src,
            "cpu_baseline": cpu, "cpu_baseline_fast": cpu_fast, "e2e": e2e, "gpu_launches": gpu_launches,
            "gpu_launches_per_step": gpu_launches / args.steps, "clocks": clk,
            "step_ms_all": [round(v, 4) for v in step_ms],
            "decode": decode, **extra,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# ---------------------------------------------------------------------------------------------
# one kernel case (profiler captures and quick timing)
# ---------------------------------------------------------------------------------------------
def run_case(a) -> int:
    """Runs one kernel case `--iters` times after two warm-up calls and prints the mean device time
    per call (CUDA events). Inputs are seeded and synthetic (weights N(0, 0.02), activations
    N(0, 1)). Examples:
        python bench.py --case gemm --m 16384 --n 5632 --k 1024
        python bench.py --case scan --b 8 --t 2048 --d 1024
        python bench.py --case block --m 16384 --d 1024 --inner 2816
        python bench.py --case decode --b 1 --d 2560 --inner 7040 --layers 4
        python bench.py --case head --b 8 --d 2560 --vocab 32000 --iters 1
    """
    import torch

    import ternary_weight_matmul_b200 as mmf

    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    dt = torch.bfloat16 if a.dtype == "bf16" else torch.float32
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    mmf.set_gemm_path({"auto": mmf.MMF_GEMM_AUTO, "tensor": mmf.MMF_GEMM_TENSOR, "simt": mmf.MMF_GEMM_SIMT}[a.engine])
    mmf.set_decode_path({"auto": mmf.MMF_DECODE_AUTO, "fused": mmf.MMF_DECODE_FUSED, "skinny": mmf.MMF_DECODE_SKINNY,
                         "block": mmf.MMF_DECODE_BLOCK}[a.decode_path])

    def blocks_of(d, inner, layers):
        shapes = {"i": (d, d), "f": (d, d), "g": (d, d), "o": (d, d), "gate": (2 * inner, d), "down": (d, inner)}
        out = []
        for _ in range(layers):
            packed = {p: mmf.pack_ternary(torch.randn(n, k, generator=g, device=dev) * 0.02) for p, (n, k) in shapes.items()}
            norms = {f"nw_{p}": torch.ones(k, device=dev) for p, (n, k) in shapes.items()}
            norms["gnorm_w"] = torch.ones(d, device=dev)
            out.append(mmf.Block(d, inner, packed, norms))
        return out

    if a.case == "gemm":
        w = mmf.pack_ternary(torch.randn(a.n, a.k, generator=g, device=dev) * 0.02)
        x = torch.randn(a.m, a.k, generator=g, device=dev).to(dt)

        def run():
            return mmf.bitlinear_fwd(x, None, w, y_dtype=dt)
        work, unit = 2.0 * a.m * a.n * a.k, "TOPS"
    elif a.case == "scan":
        zf = torch.randn(a.b, a.t, a.d, generator=g, device=dev).add_(4.0).to(dt)
        zi = torch.randn(a.b, a.t, a.d, generator=g, device=dev).to(dt)
        es = 4 if dt == torch.float32 else 2

        def run():
            return mmf.hgrn_scan(zf, zi, None, h_dtype=dt)
        work, unit = float(a.b * a.t * a.d * 3 * es), "GB/s"
    elif a.case == "norm":
        x = torch.randn(a.m, a.k, generator=g, device=dev).to(dt)
        w = mmf.pack_ternary(torch.randn(64, a.k, generator=g, device=dev) * 0.02)

        def run():
            return mmf.bitlinear_fwd(x, None, w, y_dtype=dt)
        work, unit = float(a.m * a.k * (x.element_size() + 1)), "GB/s (norm part only)"
    elif a.case == "decode":
        blocks = blocks_of(a.d, a.inner, a.layers)
        x = torch.randn(a.b, a.d, generator=g, device=dev).to(dt)
        state = torch.zeros(a.layers, a.b, a.d, device=dev)
        y = torch.empty_like(x)

        def run():
            return mmf.decode_step(blocks, x, state, out=y)
        wbytes = sum(p.codes.numel() * 4 for blk in blocks for p in blk.packed.values())
        work, unit = float(wbytes), f"GB/s (packed weights; path {mmf.decode_path(a.b, a.d, a.inner)})"
    elif a.case == "head":
        table = (torch.randn(a.vocab, a.d, generator=g, device=dev) * 0.02).to(torch.bfloat16)
        nw = torch.ones(a.d, device=dev)
        x = torch.randn(a.b, a.d, generator=g, device=dev).to(dt)
        ids = torch.empty(a.b, dtype=torch.int32, device=dev)

        def run():
            return mmf.lm_head_argmax(x, nw, table, ids_out=ids)
        work, unit = float(table.numel() * 2 * ((a.b + 127) // 128 if a.b >= 2 else 1)), "GB/s (table)"
    elif a.case == "hgrn2":
        dk = a.d // a.heads
        q = torch.randn(a.b, a.t, a.heads, dk, generator=g, device=dev).to(dt)
        f = torch.sigmoid(torch.randn(a.b, a.t, a.heads, dk, generator=g, device=dev) + 2).to(dt)
        i = torch.randn(a.b, a.t, a.heads, dk, generator=g, device=dev).to(dt)

        def run():
            return mmf.hgrn2_recurrence(q, f, i)
        work, unit = 4.0 * a.b * a.t * a.heads * dk * dk, "TFLOP/s (fp32 FMA)"
    elif a.case == "scan_bwd":
        zf = torch.randn(a.b, a.t, a.d, generator=g, device=dev).add_(2.0).to(dt)
        zi = torch.randn(a.b, a.t, a.d, generator=g, device=dev).to(dt)
        h, _ = mmf.hgrn_scan(zf, zi, None, h_dtype=dt)
        dh = torch.randn(a.b, a.t, a.d, generator=g, device=dev).to(dt)

        def run():
            return mmf.hgrn_scan_backward(zf, zi, h, dh)
        work, unit = float(6 * a.b * a.t * a.d * (4 if dt == torch.float32 else 2)), "GB/s"
    elif a.case == "lin_bwd":
        w = mmf.pack_ternary(torch.randn(a.n, a.k, generator=g, device=dev) * 0.02)
        x = torch.randn(a.m, a.k, generator=g, device=dev).to(dt)
        nw = torch.ones(a.k, device=dev)
        _, qq, deq, _ = mmf.bitlinear_fwd(x, nw, w, y_dtype=torch.float32, debug=True)
        dy = torch.randn(a.m, a.n, generator=g, device=dev).to(dt)

        def run():
            return mmf.bitlinear_backward(x, nw, w, qq, deq, dy)
        work, unit = 4.0 * a.m * a.n * a.k, "TFLOP/s (dr + dW)"
    else:  # block
        blk = blocks_of(a.d, a.inner, 1)[0]
        x = torch.randn(1, a.m, a.d, generator=g, device=dev).to(dt)

        def run():
            return mmf.block_fwd(blk, x)
        work, unit = 2.0 * a.m * (4 * a.d * a.d + 3 * a.d * a.inner), "TOPS (GEMM ops / block time)"

    for _ in range(2):
        run()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if a.case in ("decode", "head"):
        # replayed from a CUDA graph, as the decode measurement runs it (no host launch costs)
        cs = torch.cuda.Stream()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cs):
            run()
        with torch.cuda.stream(cs):
            graph.replay()
            torch.cuda.synchronize()
            s.record(cs)
            for _ in range(a.iters):
                graph.replay()
            e.record(cs)
        torch.cuda.synchronize()
    else:
        s.record()
        for _ in range(a.iters):
            run()
        e.record()
        torch.cuda.synchronize()
    st = mmf.sync_status(dev)
    ms = s.elapsed_time(e) / a.iters
    rate = work / (ms / 1e3) / (1e12 if "TOPS" in unit or "TFLOP" in unit else 1e9)
    print(f"{a.case}: {ms:.4f} ms/iter, {rate:.1f} {unit}, status {st}")
    return 0 if st == 0 else 1


def main():
    args = parse()
    if args.case:
        return run_case(args)
    wl = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, wl)
    return run_gpu(args, wl)


if __name__ == "__main__":
    sys.exit(main())
