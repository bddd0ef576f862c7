"""Run one kernel case of the library a few times, for profiler captures (ncu) and quick timing.

    python -m ternary_weight_matmul_b200.profile_cases gemm --m 16384 --n 5632 --k 1024
    python -m ternary_weight_matmul_b200.profile_cases scan --b 4 --t 8192 --d 2048
    python -m ternary_weight_matmul_b200.profile_cases block --m 16384 --d 1024 --inner 2816
    python -m ternary_weight_matmul_b200.profile_cases decode --b 1 --d 2560 --inner 7040 --layers 4
    python -m ternary_weight_matmul_b200.profile_cases head --b 8 --d 2560 --vocab 32000 --iters 1

Inputs are seeded and synthetic (weights N(0, 0.02), activations N(0, 1)); prints the mean device
time per iteration measured with CUDA events.
"""
from __future__ import annotations

import argparse

import torch

import ternary_weight_matmul_b200 as mmf


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=["gemm", "scan", "block", "norm", "decode", "head"])
    ap.add_argument("--layers", type=int, default=4)
    ap.add_argument("--m", type=int, default=16384)
    ap.add_argument("--n", type=int, default=5632)
    ap.add_argument("--k", type=int, default=1024)
    ap.add_argument("--b", type=int, default=4)
    ap.add_argument("--t", type=int, default=8192)
    ap.add_argument("--d", type=int, default=1024)
    ap.add_argument("--inner", type=int, default=2816)
    ap.add_argument("--vocab", type=int, default=32000)
    ap.add_argument("--dtype", default="bf16", choices=["bf16", "f32"])
    ap.add_argument("--iters", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=2)
    ap.add_argument("--engine", default="auto", choices=["auto", "tensor", "simt"])
    a = ap.parse_args()

    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    dt = torch.bfloat16 if a.dtype == "bf16" else torch.float32
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    mmf.set_gemm_path({"auto": mmf.MMF_GEMM_AUTO, "tensor": mmf.MMF_GEMM_TENSOR, "simt": mmf.MMF_GEMM_SIMT}[a.engine])

    if a.case == "gemm":
        w = mmf.pack_ternary(torch.randn(a.n, a.k, generator=g, device=dev) * 0.02)
        x = torch.randn(a.m, a.k, generator=g, device=dev).to(dt)
        y = torch.empty(a.m, a.n, dtype=dt, device=dev)

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
        d, inner = a.d, a.inner
        shapes = {"i": (d, d), "f": (d, d), "g": (d, d), "o": (d, d), "gate": (2 * inner, d), "down": (d, inner)}
        blocks = []
        for _ in range(a.layers):
            packed = {p: mmf.pack_ternary(torch.randn(n, k, generator=g, device=dev) * 0.02) for p, (n, k) in shapes.items()}
            norms = {f"nw_{p}": torch.ones(k, device=dev) for p, (n, k) in shapes.items()}
            norms["gnorm_w"] = torch.ones(d, device=dev)
            blocks.append(mmf.Block(d, inner, packed, norms))
        x = torch.randn(a.b, d, generator=g, device=dev).to(dt)
        state = torch.zeros(a.layers, a.b, d, device=dev)
        y = torch.empty_like(x)

        def run():
            return mmf.decode_step(blocks, x, state, out=y)
        wbytes = sum(p.codes.numel() * 4 for blk in blocks for p in blk.packed.values())
        work, unit = float(wbytes), "GB/s (packed weights)"
    elif a.case == "head":
        table = (torch.randn(a.vocab, a.d, generator=g, device=dev) * 0.02).to(torch.bfloat16)
        nw = torch.ones(a.d, device=dev)
        x = torch.randn(a.b, a.d, generator=g, device=dev).to(dt)
        ids = torch.empty(a.b, dtype=torch.int32, device=dev)

        def run():
            return mmf.lm_head_argmax(x, nw, table, ids_out=ids)
        work, unit = float(table.numel() * 2 * ((a.b + 127) // 128 if a.b >= 2 else 1)), "GB/s (table)"
    else:
        d, inner = a.d, a.inner
        shapes = {"i": (d, d), "f": (d, d), "g": (d, d), "o": (d, d), "gate": (2 * inner, d), "down": (d, inner)}
        packed = {p: mmf.pack_ternary(torch.randn(n, k, generator=g, device=dev) * 0.02) for p, (n, k) in shapes.items()}
        norms = {f"nw_{p}": torch.ones(k, device=dev) for p, (n, k) in shapes.items()}
        norms["gnorm_w"] = torch.ones(d, device=dev)
        blk = mmf.Block(d, inner, packed, norms)
        x = torch.randn(1, a.m, d, generator=g, device=dev).to(dt)

        def run():
            return mmf.block_fwd(blk, x)
        work, unit = 2.0 * a.m * (4 * d * d + 3 * d * inner), "TOPS (GEMM ops / block time)"

    for _ in range(a.warmup):
        run()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(a.iters):
        run()
    e.record()
    torch.cuda.synchronize()
    st = mmf.sync_status(dev)
    ms = s.elapsed_time(e) / a.iters
    rate = work / (ms / 1e3) / (1e12 if "TOPS" in unit else 1e9)
    print(f"{a.case}: {ms:.4f} ms/iter, {rate:.1f} {unit}, status {st}")


if __name__ == "__main__":
    main()
