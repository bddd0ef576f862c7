"""Benchmark of the HGRNBit block-stack forward on B200.

Workload (default): the 370M-shape stack, prefill forward, 24 HGRNBit blocks of hidden 1024 with
MLP gate_proj 1024->5632 and down_proj 2816->1024, vocabulary 32000 embedding, bf16 activations,
token ids uniform in [0, 32000) for batch 8 x sequence 2048 per GPU. Weights are random N(0, 0.02)
latent weights ternarised and 2-bit packed by the library. One step = one forward of the whole
stack (embedding gather + 24 blocks) over one batch.

Prints one JSON line (rank 0). --impl reference times the CPU oracle on a bounded sample of the
same workload instead. Multi-GPU runs are independent replicas (one batch per rank, no
collective on the data path); timing is the max over ranks.
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

WORKLOADS = {
    "prefill-370M": dict(d=1024, inner=2816, layers=24, vocab=32000, batch=8, seq=2048),
    "prefill-1.3B": dict(d=2048, inner=5632, layers=24, vocab=32000, batch=16, seq=2048),
}
# Autoregressive decode of the 2.7B-shape stack: a 512-token prompt (prefill, untimed) then
# decode steps with the recurrent state carried per layer, at three batch sizes.
# DRAM traffic of one ternary_gemm_tc_kernel launch (dram__bytes_read.sum + dram__bytes_write.sum,
# averaged over the 96 GEMM launches of one step) from an ncu capture of this bench's own workload;
# valid only while the kernel source is the one captured (SHA-256 prefix), else reported as null.
GEMM_TRAFFIC = {"prefill-370M": dict(bytes=78.3e6, algorithmic=115.2e6, sha256="14a6d8df0242cadf",
                                     profile="profiles/ternary_gemm_tc_kernel_prefill-370M_traffic.md")}
DECODE = dict(name="decode-2.7B", d=2560, inner=7040, layers=32, vocab=32000, prompt=512, batches=(1, 8, 64))


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
    ap.add_argument("--decode-steps", type=int, default=64)
    return ap.parse_args()


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
# CPU oracle timing (reference arm and cpu_baseline)
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


def run_decode(args, device, hbm_peak, world=1):
    """Greedy autoregressive decode throughput of the 2.7B-shape stack for each batch size: prompt
    prefill through mmf_stack_fwd (untimed; gives every layer's recurrent state and, through the
    final norm and the tied head, the first generated token), then `--decode-steps` generated
    tokens, each step = embedding gather of the current ids + mmf_decode_step + final RMSNorm,
    tied head and argmax (mmf_lm_head_argmax writes the next ids in place), replayed from a CUDA
    graph (captured after warm-up) and timed with CUDA events on the replay stream. HBM roofline:
    every step streams all packed weights and the bf16 head table (once per pass of the head: one
    row on the CUDA cores, up to 128 rows on the tensor cores). With several ranks every rank is
    a replica generating for its own sequences; the ranks meet at a barrier before each timed
    region and the step time is the slowest rank's."""
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
        out["batches"][str(B)] = decode_entry(B, ms, step_bytes, device, world, hbm_peak)
        del graph
    del blocks, table
    torch.cuda.empty_cache()
    return out


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
    blocks, table = build_model(wl, device)
    B, T, d = wl["batch"], wl["seq"], wl["d"]
    g = torch.Generator(device="cpu")
    g.manual_seed(4321 + rank)
    ids_host = torch.randint(0, wl["vocab"], (B, T), generator=g, dtype=torch.int32).pin_memory()
    ids = ids_host.to(device)
    y = torch.empty(B, T, d, dtype=torch.bfloat16, device=device)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device=device)

    def step():
        mmf.stack_fwd(blocks, ids, table, out=y)

    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        step()
    st = mmf.sync_status(device)
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up")

    # ---------------- timed region (device time, events on the launching stream)
    stream = torch.cuda.current_stream(device)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    clocks = Clocks(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(device)
    clocks.start()
    time.sleep(0.3)
    launches0 = mmf.launch_count()
    mmf.timing_enable(True)
    for i in range(args.steps):
        flush.zero_()  # write a buffer larger than L2 between steps (not timed)
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize(device)
    mmf.timing_enable(False)
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
    tokens = B * T * world
    value = replicas_throughput(B * T, world, ms_max)

    kern = {}
    for cls in ("gemm_tc", "gemm_simt", "norm_quant", "scan", "other"):
        n, kms, work = mmf.timing_read(cls)
        kern[cls] = {"launches": n, "ms": kms, "work": work}
    # our kernels launched per step: timing scopes count launches (pack uses none here)
    gpu_launches = int(launches)

    # ---------------- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        y_host = torch.empty(B, T, d, dtype=torch.bfloat16).pin_memory()
        e_s = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        e_e = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(device)
        for i in range(args.steps):
            flush.zero_()
            e_s[i].record(stream)
            ids_dev = ids_host.to(device, non_blocking=True)
            yy, _ = mmf.stack_fwd(blocks, ids_dev, table, out=y)
            y_host.copy_(yy, non_blocking=True)
            e_e[i].record(stream)
        torch.cuda.synchronize(device)
        e_ms = sum(s.elapsed_time(e) for s, e in zip(e_s, e_e)) / args.steps
        e2e = {"value": replicas_throughput(B * T, world, max_over_ranks(e_ms, device, world)), "unit": "tokens/s",
               "h2d_bytes_per_step": ids_host.numel() * 4, "d2h_bytes_per_step": y_host.numel() * 2}

    decode = None
    if not args.no_decode:  # every rank: decode replicas, timed as the slowest rank
        pp = os.path.join(ROOT, "MEASURED_PEAKS.json")
        hbm = json.load(open(pp)).get("hbm_gbs", 6650.0) if os.path.exists(pp) else 6650.0
        decode = run_decode(args, device, hbm, world)

    line = None
    if rank == 0:
        peaks = {}
        pp = os.path.join(ROOT, "MEASURED_PEAKS.json")
        if os.path.exists(pp):
            with open(pp) as fh:
                peaks = json.load(fh)
        if peaks.get("bf16_tflops_sustained"):
            int8_peak = peaks["bf16_tflops_sustained"] * INT8_OVER_BF16
            peak_src = "of measured: bf16 sustained cuBLAS x nominal int8/bf16 ratio 2"
        else:
            int8_peak = 1400.0 * INT8_OVER_BF16
            peak_src = "of fallback: 1.4 PFLOP/s bf16 sustained x nominal ratio 2"
        hbm_peak = peaks.get("hbm_gbs", 6650.0)
        tc = kern["gemm_tc"]
        achieved = (tc["work"] / (tc["ms"] / 1e3) / 1e12) if tc["ms"] > 0 else 0.0
        roofline = {"bound": "tensor", "kernel": "ternary_gemm_tc_kernel", "achieved": achieved,
                    "peak": int8_peak, "unit": "TOPS (int8)", "frac": achieved / int8_peak,
                    "peak_source": peak_src, "traffic": gemm_traffic(args.workload),
                    "traffic_source": GEMM_TRAFFIC.get(args.workload, {}).get("profile"),
                    "algorithmic_bytes_per_launch": GEMM_TRAFFIC.get(args.workload, {}).get("algorithmic"),
                    "launches": tc["launches"], "avg_launch_us": tc["ms"] / max(tc["launches"], 1) * 1e3,
                    "share_of_step": tc["ms"] / (ms * args.steps)}
        hbm_kernels = {}
        for cls in ("norm_quant", "scan", "gemm_simt", "other"):
            k = kern[cls]
            if k["launches"]:
                gbs = k["work"] / (k["ms"] / 1e3) / 1e9
                hbm_kernels[cls] = {"launches": k["launches"], "ms_total": k["ms"], "GB/s": gbs,
                                    "frac_hbm": gbs / hbm_peak, "share_of_step": k["ms"] / (ms * args.steps)}
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            v, desc, dt = oracle_sample_tokens_per_s(wl, 1024)
            cpu = {"value": v, "unit": "tokens/s", "cores": oracle_threads(), "kind": "oracle",
                   "sample": desc + f" ({dt:.1f} s)", "host_cpus": os.cpu_count()}
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "s8 x ternary -> s32 GEMM; bf16 activations, f32 reductions",
            "data": "synthetic (seeded random N(0,0.02) ternarised weights, uniform token ids)",
            "config": {"workload": args.workload, "model": "HGRNBit stack (random init)",
                       "global_batch": B * world, "seq_len": T, "hidden": d, "inner": wl["inner"],
                       "layers": wl["layers"], "vocab": wl["vocab"], "parallelism": f"replicas x{world}",
                       "l2": "flushed between steps (write of a 2x-L2 buffer, untimed)"},
            "roofline": roofline, "hbm_kernels": hbm_kernels, "hbm_peak_gbs": hbm_peak,
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": gpu_launches,
            "gpu_launches_per_step": gpu_launches / args.steps, "clocks": clk,
            "step_ms_all": [round(v, 4) for v in step_ms],
            "decode": decode,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    wl = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, wl)
    return run_gpu(args, wl)


if __name__ == "__main__":
    sys.exit(main())
