"""Benchmark of the NVFP4 verify GEMM on B200: the full 64-layer verify-pass weight stream.

Workload (the spec configuration): 64 layers x {QKV 5120->7168, O 5120->5120,
gate+up 5120->34816, down 17408->5120}, all NVFP4 (21.14 G weights, 11.89 GB of codes and
scales), each matrix with its own X (bf16, N(0,1)) and Y. Weights are drawn on the GPU
(N(0, 0.02); 0.02*t(4) for down) and packed by the library's quantiser; everything is
synthetic and seeded. One step = one pass of the whole stack at every row count M = 1..32,
one tl_nvfp4_verify_stack launch per M (the staircase). The working set (11.9 GB) is far
larger than L2, so no flush is needed between passes.

Prints ONE JSON line (rank 0). Value = algorithmic bytes of all passes / device time.
With --gpus N (torchrun), every rank runs its own replica (the path does not shard;
replicas only); value = all ranks' bytes / max-over-ranks time.

--impl reference times the CPU oracle (the only reference this workload has) on a bounded
sample of the same workload on the host cores.
"""

from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "verify-GEMM µs and HBM GB/s vs rows M=1–32; % of B200 HBM peak (1 GPU)"
LAYERS = 64
M_SWEEP = list(range(1, 33))
WORKLOAD = ("64-layer verify-pass weight stream: 64 x {QKV 5120->7168, O 5120->5120, gate+up 5120->34816, "
            "down 17408->5120}, NVFP4 (E2M1 codes, E4M3 per-16 scales, FP32 tensor scale), bf16 X/Y, "
            "one stack pass per M = 1..32")


# tensor-core paths of the library (tl_set_gemm_path), what one stack pass launches on each, and
# the arithmetic each computes in. "exact" is the default and the headline: its products are
# exact, so it meets the per-element tolerance on every input; "block-scaled" is approximate
# (X rewritten as FP4 pieces) and is reported only as a separately labelled run.
PATHS = {"exact": 2, "bf16-exact": 1, "block-scaled": 0}
KERNELS = {"exact": "x_prep_kernel + gemm_ex_kernel<NX> + fallback_rows_kernel (three launches per stack pass, "
                    "timed together)",
           "bf16-exact": "gemm_tc_kernel<NX, bf16> (one launch per stack pass)",
           "block-scaled": "x_split_kernel + gemm_bs_kernel (two launches per stack pass, timed together)"}
LAUNCHES = {"exact": 3, "bf16-exact": 1, "block-scaled": 2}
DTYPES = {"exact": "f16", "bf16-exact": "bf16", "block-scaled": "fp4"}
ARITHMETIC = {
    "exact": "f16 x f16 tensor-core products, fp32 accumulate; operands are exact copies of the bf16 X (each row "
             "times a power of two) and of W' = e2m1 * e4m3, so every product is exact",
    "bf16-exact": "bf16 x bf16 tensor-core products, fp32 accumulate; X as given, W' = e2m1 * e4m3 exact in bf16",
    "block-scaled": "APPROXIMATE: e2m1 x e2m1 block-scaled tensor-core products (e4m3 scales per 16), fp32 "
                    "accumulate; X rewritten as four FP4 pieces, not exact",
}


def stack_shapes():
    import synth
    out = []
    for layer in range(LAYERS):
        for j, (name, K, N) in enumerate(synth.LAYER_SHAPES):
            out.append((layer, j, name, N, K, synth.LAYER_DISTS[name]))
    return out


def w_bytes(shapes):
    return sum(N * K // 2 + N * K // 16 + 4 for (_, _, _, N, K, _) in shapes)


def pass_bytes(shapes, M):
    """Algorithmic bytes of one stack pass: every code, scale, X and Y element once."""
    return w_bytes(shapes) + sum(2 * M * K + 2 * M * N for (_, _, _, N, K, _) in shapes)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# the device code of each path: a recorded DRAM figure holds while these files are unchanged
PATH_SOURCES = {
    "exact": ("gemm_ex.cuh", "gemm_tc.cuh", "xprep.cuh", "ptx.cuh", "nvfp4_format.cuh"),
    "bf16-exact": ("gemm_tc.cuh", "ptx.cuh", "nvfp4_format.cuh"),
    "block-scaled": ("gemm_bs.cuh", "xsplit.cuh", "ptx.cuh", "nvfp4_format.cuh"),
}


def source_hash(path="exact"):
    h = hashlib.sha256()
    for f in PATH_SOURCES[path]:
        h.update(open(os.path.join(ROOT, "nvfp4_weight_gemm_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(shapes, path):
    """DRAM bytes of the mean stack pass (M = 1..32), from the committed ncu record of the pass's
    kernels at several M (ratio to the algorithmic bytes, linear in between), if it was taken on
    this source and path (None otherwise)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    if d.get("source_hash") != source_hash(path) or not d.get("kernels", "").startswith(KERNELS[path].split(" (")[0]):
        return None
    pts = sorted((int(m), v["ratio"]) for m, v in d["per_M"].items())

    def ratio(M):
        for (m0, r0), (m1, r1) in zip(pts, pts[1:]):
            if m0 <= M <= m1:
                return r0 + (r1 - r0) * (M - m0) / (m1 - m0)
        return pts[0][1] if M < pts[0][0] else pts[-1][1]
    return round(sum(ratio(M) * pass_bytes(shapes, M) for M in M_SWEEP) / len(M_SWEEP))


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,"
              "power.limit,temperature.gpu,temperature.memory,clocks.mem")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"tl_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        def num(i):
            return [float(r[i]) for r in rows if len(r) > i and r[i].replace(".", "").isdigit()]
        pw, lim, tg, tm, mem = num(3), num(9), num(10), num(11), num(12)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows), "power_w_max": max(pw) if pw else None,
                "power_limit_w": max(lim) if lim else None, "temp_gpu_c_max": max(tg) if tg else None,
                "temp_mem_c_max": max(tm) if tm else None, "mem_mhz": statistics.median(mem) if mem else None}


# --------------------------------------------------------------------------- CPU oracle sample

def cpu_sample(rows_per_shape: int, M: int):
    """Time the CPU oracle on `rows_per_shape` weight rows of each of the four layer shapes at M rows.

    Returns (bytes, seconds, threads). The oracle is used as it stands (fp64, OpenMP over rows)."""
    import oracle
    import synth
    oracle.build()
    total_b, total_t = 0, 0.0
    for j, (name, K, N) in enumerate(synth.LAYER_SHAPES):
        w = synth.w_f32(rows_per_shape, K, seed=0, tensor_id=j, dist=synth.LAYER_DISTS[name])
        codes, scales, g = oracle.quantize(w)
        x = synth.x_bf16(M, K, seed=0, tensor_id=synth.X_ID_BASE + j)
        t0 = time.perf_counter()
        oracle.gemm(x, codes, scales, g)
        total_t += time.perf_counter() - t0
        total_b += rows_per_shape * K // 2 + rows_per_shape * K // 16 + 2 * M * K + 2 * M * rows_per_shape
    return total_b, total_t, oracle.num_threads()


CPU_ROWS = 192
CPU_SAMPLE_DESC = (f"{CPU_ROWS} weight rows of each layer shape (QKV, O, gate+up, down), full K, at M = 32: "
                   f"fp64 oracle GEMM, GB/s over the same algorithmic bytes")


def arm_config(path, world):
    """The `config` of the bench line; the reference arm prints the same one (its sample of the
    workload is named in its `cpu_baseline`)."""
    shapes = stack_shapes()
    return {"workload": WORKLOAD, "path": path, "arithmetic": ARITHMETIC[path], "matrices": len(shapes),
            "weights": sum(N * K for (_, _, _, N, K, _) in shapes), "w_bytes": w_bytes(shapes),
            "M": "1..32 (one pass each per step)", "l2": "working set 11.9 GB >> 126 MB L2; no flush needed",
            "parallelism": f"replicas x{world}"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    for _ in range(args.warmup):
        cpu_sample(CPU_ROWS // 4, 32)
    byts, secs = 0, 0.0
    threads = 1
    for _ in range(args.steps):
        b, s, threads = cpu_sample(CPU_ROWS, 32)
        byts += b
        secs += s
    value = byts / secs / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": arm_config(args.path, int(os.environ.get("WORLD_SIZE", "1"))),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": CPU_SAMPLE_DESC},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- replicas

def max_over_ranks(values, device, world):
    """Element-wise maximum of per-rank timings over all ranks (every rank must call it)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_gbs(world, bytes_per_rank, ms):
    """Whole-job GB/s of `world` replicas: every rank's bytes over the slowest rank's time."""
    return world * bytes_per_rank / (ms * 1e-3) / 1e9


# --------------------------------------------------------------------------- GPU arm

def build_stack(dev, seed=0):
    """Draw and pack every weight of the stack on `dev`. Returns [(codes, scales, g, N, K)]."""
    import torch
    import nvfp4_weight_gemm_b200 as tl
    import synth
    out = []
    for (layer, j, name, N, K, dist) in stack_shapes():
        w = synth.w_f32_torch(N, K, seed, layer * 4 + j, dev, dist)
        codes, scales, g = tl.quantize(w)
        del w
        out.append((codes, scales, g, N, K))
    torch.cuda.synchronize()
    return out


def main_gpu(args):
    import torch
    import torch.distributed as dist
    import nvfp4_weight_gemm_b200 as tl
    import synth
    from nvfp4_weight_gemm_b200 import build as tlbuild

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if rank == 0:
        tlbuild.build()
    if world > 1:
        dist.barrier()
    tl.init(local)
    tl.set_gemm_path(PATHS[args.path])
    launches_per_pass = LAUNCHES[args.path]

    shapes = stack_shapes()
    stack = build_stack(dev, seed=rank)
    Mmax = max(M_SWEEP)
    xs = [synth.x_bf16_torch(Mmax, K, rank, synth.X_ID_BASE + i, dev) for i, (_, _, _, N, K) in enumerate(stack)]
    ys = [torch.empty((Mmax, N), dtype=torch.bfloat16, device=dev) for (_, _, _, N, K) in stack]
    stream = torch.cuda.Stream(device=dev)

    # one plan per M: X/Y views of the first M rows (row-major prefixes are contiguous)
    plans = {M: tl.Plan([(c, s, g, xs[i][:M], ys[i][:M]) for i, (c, s, g, N, K) in enumerate(stack)], M)
             for M in M_SWEEP}

    def run_pass(M):
        plans[M].run(stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(max(1, args.warmup)):
            for M in M_SWEEP:
                run_pass(M)
    stream.synchronize()
    tl.check_device_error(stream)

    # ---- timed region: device events around every launch, on the launching stream
    n_launch = args.steps * len(M_SWEEP)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_launch)]
    clk = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clk.start()
    time.sleep(0.3)
    t_start = torch.cuda.Event(enable_timing=True)
    t_stop = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    i = 0
    for _ in range(args.steps):
        for M in M_SWEEP:
            ev[i][0].record(stream)
            run_pass(M)
            ev[i][1].record(stream)
            i += 1
    t_stop.record(stream)
    stream.synchronize()
    clocks = clk.stop()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    tl.check_device_error(stream)
    total_ms = t_start.elapsed_time(t_stop)
    per = [e0.elapsed_time(e1) for e0, e1 in ev]
    per_M = {M: statistics.median(per[j::len(M_SWEEP)]) for j, M in enumerate(M_SWEEP)}
    per_M_min = {M: min(per[j::len(M_SWEEP)]) for j, M in enumerate(M_SWEEP)}
    bytes_step = sum(pass_bytes(shapes, M) for M in M_SWEEP)
    launch_ms_sum = sum(per)

    # ---- end to end through the C ABI with host buffers (copies inside the timed region):
    # per M, a plan whose X_i / Y_i are packed back to back in one device buffer each
    xtot = sum(Mmax * K for (_, _, _, N, K) in stack)
    ytot = sum(Mmax * N for (_, _, _, N, K) in stack)
    x_host = torch.empty(xtot, dtype=torch.bfloat16).pin_memory()
    off = 0
    for x in xs:
        x_host[off:off + x.numel()].copy_(x.reshape(-1).cpu())
        off += x.numel()
    y_host = torch.empty(ytot, dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty(xtot, dtype=torch.bfloat16, device=dev)
    y_dev = torch.empty(ytot, dtype=torch.bfloat16, device=dev)
    e2e_plans = {}
    for M in M_SWEEP:
        ents, xo, yo = [], 0, 0
        for (c, s, g, N, K) in stack:
            ents.append((c, s, g, x_dev[xo:xo + M * K].view(M, K), y_dev[yo:yo + M * N].view(M, N)))
            xo += M * K
            yo += M * N
        e2e_plans[M] = tl.Plan(ents, M)
    e2e_h2d = sum(2 * M * K for M in M_SWEEP for (_, _, _, N, K) in stack)
    e2e_d2h = sum(2 * M * N for M in M_SWEEP for (_, _, _, N, K) in stack)

    def e2e_step():
        for M in M_SWEEP:
            e2e_plans[M].run_host(x_host, y_host, stream=stream)

    e2e_step()
    stream.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    e0.record(stream)
    e2e_steps = max(1, args.steps // 2)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    stream.synchronize()
    tl.check_device_error(stream)
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    for pl in e2e_plans.values():
        pl.close()

    # ---- M-invariance: sampled rows i at M=k against the same row computed alone (M=1)
    inv = {}
    for k in (8, 32):
        plans[k].run(stream=stream)
        stream.synchronize()
        yk = [y[:k].clone() for y in ys]
        same = total = 0
        for i_row in sorted({0, k // 2, k - 1}):
            p1 = tl.Plan([(c, s, g, xs[i][i_row:i_row + 1], ys[i][:1]) for i, (c, s, g, N, K) in enumerate(stack)], 1)
            p1.run(stream=stream)
            stream.synchronize()
            p1.close()
            for i in range(len(stack)):
                same += int(torch.equal(ys[i][0], yk[i][i_row]))
                total += 1
        inv[str(k)] = same / total
    tl.check_device_error(stream)

    # ---- the benchmarked stack against the oracle, sampled: every matrix, at M = 8, 16, 24, 32
    parity = sampled_parity(tl, stack, xs, ys, plans, stream, rank) if rank == 0 else None

    # ---- the FP8 output head after the stack: vocabulary-sized logits + greedy top-2 per M, and
    # the closed-form commit of the accepted path through the GDN layers' states (secondary
    # figures: a failure here is reported in the line instead of losing it)
    head = gdn = None
    if rank == 0:
        try:
            head = head_figure(tl, dev, stream, rank)
        except Exception as exc:
            head = {"error": f"{type(exc).__name__}: {str(exc)[:300]}"}
        try:
            gdn = gdn_figure(tl, dev, stream, rank)
        except Exception as exc:
            gdn = {"error": f"{type(exc).__name__}: {str(exc)[:300]}"}

    # ---- reduce over ranks: max time, summed bytes
    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], dev, world)

    if rank == 0:
        peak, peak_kind = load_peaks()
        value = job_gbs(world, bytes_step * args.steps, total_ms)
        achieved = bytes_step * args.steps / (launch_ms_sum * 1e-3) / 1e9
        # per launch, like `achieved`: DRAM bytes of the mean stack pass
        traffic = profiled_traffic(shapes, args.path)
        stair = {}
        for M in M_SWEEP:
            gbs = pass_bytes(shapes, M) / (per_M[M] * 1e-3) / 1e9
            stair[str(M)] = {"us": round(per_M[M] * 1e3, 1), "us_min": round(per_M_min[M] * 1e3, 1),
                             "gbs": round(gbs, 1), "frac": round(gbs / peak, 4),
                             "w_only_gbs": round(w_bytes(shapes) / (per_M[M] * 1e-3) / 1e9, 1)}
        cb, cs, cthreads = cpu_sample(CPU_ROWS, 32)
        # what this staircase implies for the draft-tree size (host-side summary, after timing)
        try:
            from nvfp4_weight_gemm_b200 import staircut
            cut = staircut.report(staircut.Staircase({M: per_M[M] for M in M_SWEEP}))
        except Exception as exc:  # a summary only: it never fails the run
            cut = {"error": str(exc)[:200]}
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": DTYPES[args.path], "data": "synthetic",
            "config": arm_config(args.path, world),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": traffic, "peak_kind": peak_kind,
                         "kernel": KERNELS[args.path]},
            "staircase": stair,
            "min_frac_over_M": round(min(v["frac"] for v in stair.values()), 4),
            "m_invariance_row_fraction": inv,
            "parity_sampled": parity,
            "staircut": cut,
            "fp8_head": head,
            "gdn_commit": gdn,
            "cpu_baseline": {"value": round(cb / cs / 1e9, 4), "unit": "GB/s", "cores": cthreads, "kind": "oracle",
                             "sample": CPU_SAMPLE_DESC},
            "e2e": {"value": round(job_gbs(world, bytes_step, e2e_ms), 1), "unit": "GB/s",
                    "h2d_bytes_per_step": e2e_h2d, "d2h_bytes_per_step": e2e_d2h},
            "gpu_launches": n_launch * launches_per_pass,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    for pl in plans.values():
        pl.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if parity is not None and parity["outside"] > 0:
        print(f"sampled parity: {parity['outside']} of {parity['checked']} outputs outside the tolerance",
              file=sys.stderr, flush=True)
        return 1
    if gdn is not None and gdn.get("parity_sampled", {}).get("outside", 0) > 0:
        print(f"GDN commit sampled parity: {gdn['parity_sampled']['outside']} heads outside the bar",
              file=sys.stderr, flush=True)
        return 1
    if head is not None and head.get("parity_sampled", {}).get("outside", 0) > 0:
        print(f"FP8 head sampled parity: {head['parity_sampled']['outside']} logits outside the tolerance",
              file=sys.stderr, flush=True)
        return 1
    return 0


GDN_H, GDN_D, GDN_NODES = 48 * 32, 128, 32   # 48 GDN layers x 32 heads of 128 x 128 states; a 32-node tree
GDN_L = (1, 4, 8, 16, 32)
FP32_FMA_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12   # 148 SMs x 128 fp32 FMA lanes x 2 flops at 1,965 MHz


def gdn_figure(tl, dev, stream, rank):
    """Time tl_gdn_commit over 1,536 heads of 128 x 128 fp32 states for accepted paths of L = 1..32
    tokens, CUDA events on the launching stream, with a 256 MB write between launches so the
    100 MB of states come from HBM every time; then check 4 heads against the oracle."""
    import numpy as np
    import torch
    import oracle
    import synth
    peak, _ = load_peaks()
    S0, K, V, a, b = synth.gdn_inputs_torch(GDN_H, GDN_D, GDN_D, GDN_NODES, rank, dev)
    state = S0.clone()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    per_L = {}
    with torch.cuda.stream(stream):
        for L in GDN_L:
            path = list(range(L))
            for _ in range(3):
                tl.gdn_commit(state, K, V, a, b, path, stream=stream)
            times = []
            for _ in range(10):
                flush.fill_(1)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                tl.gdn_commit(state, K, V, a, b, path, stream=stream)
                e1.record(stream)
                times.append((e0, e1))
            stream.synchronize()
            ms = statistics.median(e0.elapsed_time(e1) for e0, e1 in times)
            byts = 2 * GDN_H * GDN_D * GDN_D * 4 + L * GDN_H * (2 * GDN_D + 2) * 4
            flops = 4 * GDN_H * GDN_D * GDN_D * L + GDN_H * L * L * GDN_D
            per_L[str(L)] = {"us": round(ms * 1e3, 1), "gbs": round(byts / (ms * 1e-3) / 1e9, 1),
                             "frac_hbm": round(byts / (ms * 1e-3) / 1e9 / peak, 4),
                             "tflops": round(flops / (ms * 1e-3) / 1e12, 2),
                             "frac_fp32_fma": round(flops / (ms * 1e-3) / 1e12 / FP32_FMA_PEAK_TFLOPS, 4)}
        # sampled parity: the longest path from the initial states, 4 heads
        state.copy_(S0)
        path = [0, 2, 3, 5, 8, 9, 13, 14, 17, 19, 20, 24, 26, 27, 30, 31]
        tl.gdn_commit(state, K, V, a, b, path, stream=stream)
        stream.synchronize()
    tl.check_device_error(stream)
    heads = [0, 511, 1024, GDN_H - 1]
    outside = 0
    S0h, Kh, Vh, ah, bh = (t.cpu().numpy() for t in (S0, K, V, a, b))
    got = state.cpu().numpy().astype(np.float64)
    for h in heads:
        Kp, Vp, ap, bp = oracle.gdn_path_inputs(Kh[:, h], Vh[:, h], ah[:, h], bh[:, h], path)
        ref = oracle.gdn_commit_closed_form(S0h[h], Kp, Vp, ap, bp)
        outside += int(np.abs(got[h] - ref).max() > 1e-4 * max(1.0, float(np.abs(ref).max())))
    return {"heads": GDN_H, "d_k": GDN_D, "d_v": GDN_D, "tree_nodes": GDN_NODES, "per_L": per_L,
            "bytes": "2 * H * d_v * d_k * 4 (state in and out) + L * H * (d_k + d_v + 2) * 4 per commit",
            "flops": "4 * H * d_v * d_k * L + H * L^2 * d_k", "fp32_fma_peak_tflops": round(FP32_FMA_PEAK_TFLOPS, 1),
            "kernel": "gdn_commit_kernel<128, 128> (one launch)",
            "parity_sampled": {"heads": len(heads), "outside": outside,
                               "sample": "4 heads after a 16-token path, vs the fp64 oracle (bar 1e-4 of the state)"}}


HEAD_N, HEAD_K = 151936, 5120     # a vocabulary-sized head on the stack's hidden size
HEAD_M = (1, 8, 16, 17, 24, 32)
HEAD_REPS = 20


def head_bytes(M):
    """Algorithmic bytes of one head call: E4M3 weights, per-row scales, X, fp32 logits, top-2 records."""
    return HEAD_N * HEAD_K + 4 * HEAD_N + 2 * M * HEAD_K + 4 * M * HEAD_N + 16 * M


def head_figure(tl, dev, stream, rank):
    """Time tl_fp8_head (X prep, head GEMM, and one tail launch for fp64 rows and the top-2: three launches) at a
    151,936 x 5,120 FP8 head with per-row scales, per M, with CUDA events on the launching stream
    (the 0.78 GB weight is over six times L2, so no flush), then check sampled logits against the
    oracle and the top-2 against the kernel's own logits."""
    import numpy as np
    import torch
    import oracle
    import synth
    peak, _ = load_peaks()
    w = synth.w_f32_torch(HEAD_N, HEAD_K, rank, 9000, dev)
    sc = (w.abs().amax(dim=1) / 448.0).clamp_min(1e-30)
    wq = (w / sc[:, None]).to(torch.float8_e4m3fn).view(torch.uint8).contiguous()
    sc = sc.float().contiguous()
    del w
    torch.cuda.empty_cache()
    per_M = {}
    with torch.cuda.stream(stream):
        x = synth.x_bf16_torch(max(HEAD_M), HEAD_K, rank, synth.X_ID_BASE + 9000, dev)
        logits = torch.empty((max(HEAD_M), HEAD_N), dtype=torch.float32, device=dev)
        for M in HEAD_M:
            for _ in range(3):
                tl.fp8_head(x[:M], wq, sc, logits=logits[:M], stream=stream)
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(HEAD_REPS)]
            for e0, e1 in evs:
                e0.record(stream)
                tl.fp8_head(x[:M], wq, sc, logits=logits[:M], stream=stream)
                e1.record(stream)
            stream.synchronize()
            ms = statistics.median(e0.elapsed_time(e1) for e0, e1 in evs)
            gbs = head_bytes(M) / (ms * 1e-3) / 1e9
            per_M[str(M)] = {"us": round(ms * 1e3, 1), "gbs": round(gbs, 1), "frac": round(gbs / peak, 4)}
        # sampled parity at M = 32: 512 seeded columns + the last 16, every row
        M = max(HEAD_M)
        lg, top2 = tl.fp8_head(x[:M], wq, sc, logits=logits[:M], stream=stream)
        stream.synchronize()
    tl.check_device_error(stream)
    rng = np.random.default_rng(9000)
    cols = np.unique(np.concatenate([rng.integers(0, HEAD_N, 512), np.arange(HEAD_N - 16, HEAD_N)]))
    idx = torch.from_numpy(cols).to(dev)
    w_s = wq.index_select(0, idx).cpu().numpy()
    s_s = sc.index_select(0, idx).cpu().numpy().astype(np.float64)
    xb = x[:M].cpu().view(torch.int16).numpy().view(np.uint16)
    ref = oracle.fp8_head_logits(xb, w_s, s_s)
    table = np.array([oracle.e4m3_decode(b) for b in range(256)], dtype=np.float64)
    xa = np.abs((xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64))
    tol = 1e-3 * (xa @ np.abs(np.nan_to_num(table[w_s])).T) * np.abs(s_s)[None, :] + 2.0 ** -22 * np.abs(ref)
    got = lg.index_select(1, idx).cpu().numpy().astype(np.float64)
    with np.errstate(invalid="ignore"):
        outside = int((~(np.abs(got - ref) <= tol)).sum())
    tok, t1, t2, gap = tl.head_top2_fields(top2)
    o_idx, o_t1, o_t2, _ = oracle.greedy_top2(lg.cpu().numpy().astype(np.float64))
    top2_ok = bool(np.array_equal(tok, o_idx) and np.array_equal(t1, o_t1) and np.array_equal(t2, o_t2))
    outside += 0 if top2_ok else 1
    return {"N": HEAD_N, "K": HEAD_K, "weights": "E4M3, per-row fp32 scale", "per_M": per_M,
            "min_frac_over_M": round(min(v["frac"] for v in per_M.values()), 4),
            "bytes": "N*K + 4N + 2MK + 4MN + 16M per call",
            "kernels": "x_prep_kernel + gemm_head_kernel<NX> + head_tail_kernel (timed together)",
            "gap_ulp_at_M32": [round(float(v), 3) for v in gap],
            "parity_sampled": {"checked": int(got.size), "outside": outside, "top2_matches_own_logits": top2_ok,
                               "sample": "528 weight rows (512 seeded + last 16), all 32 rows, vs fp64 oracle"}}


PARITY_M = (8, 16, 24, 32)
PARITY_ROWS = 32   # random weight rows per matrix, plus its last 16


def sampled_parity(tl, stack, xs, ys, plans, stream, rank):
    """Every matrix of the benchmarked stack at M = 8, 16, 24, 32 against the fp64 oracle:
    PARITY_ROWS seeded weight rows plus the last 16 rows of each matrix (their codes and scales
    gathered on the device and copied out), all M rows of X; element by element at the stated
    tolerance. Returns {"checked", "outside", "worst_excess"} (outputs, outputs outside, and the
    largest |y - y_ref| - tol seen)."""
    import numpy as np
    import torch
    import oracle
    oracle.build()
    rng = np.random.default_rng(1234 + rank)
    xs_host = [x.view(torch.int16).cpu().numpy().view(np.uint16) for x in xs]
    checked = outside = 0
    worst = -np.inf
    for M in PARITY_M:
        plans[M].run(stream=stream)
        stream.synchronize()
        for i, (c, s, g, N, K) in enumerate(stack):
            rows = np.unique(np.concatenate([rng.integers(0, N, PARITY_ROWS), np.arange(N - 16, N)]))
            idx = torch.from_numpy(rows).to(c.device)
            codes = c.index_select(0, idx).cpu().numpy()
            scales = s.index_select(0, idx).cpu().numpy()
            y = ys[i][:M].index_select(1, idx).float().cpu().numpy().astype(np.float64)
            y_ref, a_ref = oracle.gemm(np.ascontiguousarray(xs_host[i][:M]), codes, scales, g)
            tol = 1e-3 * a_ref + 2.0 ** -8 * np.abs(y_ref)
            with np.errstate(invalid="ignore"):
                err = np.abs(y - y_ref)
                bad = ~(err <= tol)
            checked += bad.size
            outside += int(bad.sum())
            worst = max(worst, float(np.nanmax(np.where(np.isfinite(err), err - tol, np.inf))))
    return {"checked": checked, "outside": outside, "worst_excess": worst,
            "sample": f"{PARITY_ROWS} seeded + last 16 weight rows of every matrix, all M rows, M = "
                      + ", ".join(str(m) for m in PARITY_M)}


def run_profile_case(args):
    """Small case for ncu: one matrix (--profile-matrix NxK), the first L layers of the stack
    (--profile-layers L), `--reps` launches of one plan at --M rows; or `--reps` calls of the FP8
    output head (--profile-head) at --M rows.

    Inputs are drawn and packed on the device like the stack's; prints one summary line."""
    import torch
    import nvfp4_weight_gemm_b200 as tl
    import synth
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    tl.init(0)
    tl.set_gemm_path(PATHS[args.path])
    if args.profile_head:
        w = synth.w_f32_torch(HEAD_N, HEAD_K, 0, 9000, dev)
        sc = (w.abs().amax(dim=1) / 448.0).clamp_min(1e-30)
        wq = (w / sc[:, None]).to(torch.float8_e4m3fn).view(torch.uint8).contiguous()
        sc = sc.float().contiguous()
        del w
        x = synth.x_bf16_torch(args.M, HEAD_K, 0, synth.X_ID_BASE + 9000, dev)
        for _ in range(args.reps):
            tl.fp8_head(x, wq, sc)
        torch.cuda.synchronize()
        tl.check_device_error()
        print(json.dumps({"profile_case": f"FP8 head {HEAD_N}x{HEAD_K}", "w_bytes": HEAD_N * HEAD_K, "M": args.M,
                          "reps": args.reps}), flush=True)
        return 0
    if args.profile_matrix:
        N, K = (int(v) for v in args.profile_matrix.lower().split("x"))
        shapes = [(N, K, "normal")]
        case = f"{N}x{K}"
    else:
        shapes = [(N, K, dist) for (layer, j, name, N, K, dist) in stack_shapes() if layer < args.profile_layers]
        case = f"{args.profile_layers} layers"
    ents = []
    for i, (N, K, dist) in enumerate(shapes):
        w = synth.w_f32_torch(N, K, 0, i, dev, dist)
        codes, scales, g = tl.quantize(w)
        del w
        x = synth.x_bf16_torch(args.M, K, 0, synth.X_ID_BASE + i, dev)
        ents.append((codes, scales, g, x, torch.empty((args.M, N), dtype=torch.bfloat16, device=dev)))
    plan = tl.Plan(ents, args.M)
    for _ in range(args.reps):
        plan.run()
    torch.cuda.synchronize()
    tl.check_device_error()
    plan.close()
    wb = sum(N * K // 2 + N * K // 16 for (N, K, _) in shapes)
    print(json.dumps({"profile_case": case, "matrices": len(shapes), "w_bytes": wb, "M": args.M, "reps": args.reps,
                      "path": args.path}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--profile-matrix", default=None, help="NxK: run one matrix --reps times (for ncu)")
    ap.add_argument("--profile-layers", type=int, default=0, help="L: run the first L layers of the stack (for ncu)")
    ap.add_argument("--profile-head", action="store_true", help="run the FP8 output head --reps times (for ncu)")
    ap.add_argument("--M", type=int, default=32)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--path", default="exact", choices=sorted(PATHS),
                    help="tensor-core path: exact (default; exact f16 operands), bf16-exact, or block-scaled "
                         "(approximate)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.profile_matrix or args.profile_layers or args.profile_head:
        return run_profile_case(args)
    return main_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
