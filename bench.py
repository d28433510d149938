#!/usr/bin/env python
"""DF11 decode benchmark on B200.

One step = one decode launch (df11_decode_block_batch) of a whole
transformer block: by default the seven matrices of the Llama-3-70B-shaped
block (855,638,016 BF16 weights, per-matrix codebooks), compressed by this
library from the seeded synthetic weights of ``workloads``.

Prints ONE JSON line (rank 0).  ``value`` is decoded BF16 output in GB/s
(2 bytes per weight, 1e9 bytes) summed over all ranks; each rank decodes its
own replica of the block (independent work, no collective on the data path:
weak scaling).  Extra keys: roofline of the decode kernel against the
measured HBM copy bandwidth, compression ratio, the oracle's CPU decode rate
on a bounded sample, an end-to-end figure through the C ABI with host
buffers, clocks sampled during the timed region.

``--impl reference`` times the CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "DF11 decode output BF16 GB/s & % of HBM roofline (bit-exact); ratio"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0  # the fallback dense BF16 figure (burst)
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "decode_idx_kernel_traffic.txt")
KERNEL_SOURCE = os.path.join(ROOT, "lossless_bf16_weight_df11_b200", "csrc", "df11_kernels.cu")
ORACLE_SAMPLE = ("q", "o", "k", "v", "gate")
CAP = 11  # code-length cap of the benchmarked codebooks: DF11_TABLE_BITS, the decode table's reach
L2_FLUSH_BYTES = 256 << 20  # written between timed launches of inputs that fit the 126 MB L2


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", type=int, default=5, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--impl", default="df11", choices=["df11", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-verify", action="store_true")
    ap.add_argument("--cap32", type=int, default=1, help="also time the block coded with cap 32")
    ap.add_argument("--encode-steps", type=int, default=3,
                    help="passes of the device-only encode timing (0: skip)")
    ap.add_argument("--matmul-steps", type=int, default=10,
                    help="steps of the fused decode -> matmul timing (0: skip)")
    ap.add_argument("--rans-steps", type=int, default=10,
                    help="decode launches of the block coded with the rANS variant (0: skip)")
    ap.add_argument("--block-steps", type=int, default=5,
                    help="steps of the DF11 transformer-block forward timing (0: skip)")
    ap.add_argument("--config-steps", type=int, default=10,
                    help="decode launches timed on each of the other workloads (0: skip)")
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(x: float, dist=None, device="cpu") -> float:
    """The largest value of x over all ranks (the slowest rank's time); x
    itself on a single process.  Every rank must call it at the same point."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def measured_tensor_peak():
    """Dense BF16 tensor-core peak (TFLOP/s) of this machine's B200s: the burst
    figure, for a kernel timed alone."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


DECODE_BEGIN = "// ============================================================ decode"
DECODE_END = "// ============================================================ segment decoder"


def kernel_hash() -> str:
    """Fingerprint of the indexed decoder's code (the decode section of
    df11_kernels.cu, up to the segment decoder, without comments), so that a
    stored traffic figure is used only for the kernel it was measured on."""
    with open(KERNEL_SOURCE, encoding="utf-8") as f:
        src = f.read()
    a, b = src.find(DECODE_BEGIN), src.find(DECODE_END)
    section = src[a:b] if 0 <= a < b else src
    # the code alone: line comments and whitespace do not change the kernel
    code = " ".join(re.sub(r"//[^\n]*", "", section).split())
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def profiled_traffic(workload_name: str):
    """DRAM bytes per decode launch from a committed ncu summary, if it was
    taken on the current kernel source; else None."""
    try:
        kv = {}
        for line in open(PROFILE_TRAFFIC):
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
        if kv.get("kernel_sha") != kernel_hash() or kv.get("workload") != workload_name:
            return None
        return int(float(kv["traffic_bytes_per_launch"]))
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi sampled every 200 ms while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def oracle_decode_rate(mats_np, names):
    """The CPU oracle (bit-serial, one thread) decoding a bounded sample of the
    workload: (GB/s of BF16 output, seconds, weights)."""
    import oracle
    encs = [oracle.encode(x, cap=CAP) for x in mats_np]
    t0 = time.perf_counter()
    for x, enc in zip(mats_np, encs):
        out = oracle.decode(enc)
        assert np.array_equal(out, x.reshape(-1))
    dt = time.perf_counter() - t0
    n = sum(x.size for x in mats_np)
    return 2 * n / dt / 1e9, dt, n


def cpu_info():
    """Host cores this process may use and the CPU model."""
    try:
        usable = len(os.sched_getaffinity(0))
    except Exception:
        usable = os.cpu_count() or 1
    model = None
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                model = ln.split(":", 1)[1].strip()
                break
    except Exception:
        pass
    return {"nproc": usable, "cpu_model": model}


CPU_SAMPLE = 1 << 23  # weights per matrix sample of the oracle's per-config timings


def cpu_baseline_plan(samples):
    """The oracle (plain C, bit-serial, one thread per call) on bounded samples
    of every workload: encode (histogram, codebook, bitstream) and decode on
    one core, and, for the two transformer blocks, one matrix per thread on
    min(7, nproc) cores.  samples: {workload id: [uint16 arrays]}, at most
    CPU_SAMPLE weights each.  Rates in GB/s of BF16 (input for encode,
    output for decode)."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    info = cpu_info()
    out = {"cores_available": info["nproc"], "cpu_model": info["cpu_model"], "configs": {}}
    for wid, mats in samples.items():
        x = mats[0]
        t0 = time.perf_counter()
        enc = oracle.encode(x, cap=CAP)
        t1 = time.perf_counter()
        y = oracle.decode(enc)
        t2 = time.perf_counter()
        assert np.array_equal(y, x)
        row = {"sample": f"{x.size} weights of {workloads.workload_name(wid)}",
               "encode_GBps_1core": 2 * x.size / (t1 - t0) / 1e9,
               "decode_GBps_1core": 2 * x.size / (t2 - t1) / 1e9}
        if len(mats) > 1:
            threads = max(1, min(7, info["nproc"], len(mats)))

            def one(m):
                e = oracle.encode(m, cap=CAP)
                return oracle.decode(e).size

            t0 = time.perf_counter()
            with ThreadPoolExecutor(threads) as ex:
                done = sum(ex.map(one, mats[:threads]))
            dt = time.perf_counter() - t0
            row["multicore"] = {"threads": threads, "weights": done,
                                "encode_plus_decode_s": dt,
                                "decode_side_GBps": 2 * done / dt / 1e9,
                                "what": "one matrix sample per thread, each encoded then decoded"}
        out["configs"][workloads.workload_name(wid)] = row
    return out


def time_configs(torch, df11, codec, dev, steps, warmup, peak, peak_kind, skip_wid, skip_xs):
    """Decode of every other workload in one launch per step: median launch
    time over `steps` launches, each preceded by a write of L2_FLUSH_BYTES (so
    inputs that fit the 126 MB L2 are read from HBM), with its roofline and
    compression ratio.  Returns ({workload: line}, {workload id: CPU samples})."""
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    lines, samples = {}, {}
    for wid in (1, 2, 3, 4, 5):
        if wid == skip_wid:  # the main workload: timed already, its matrices at hand
            samples[wid] = [x.reshape(-1)[:CPU_SAMPLE] for x in skip_xs]
            continue
        mats_def = workloads.WORKLOADS[wid][1]
        xs = [workloads.matrix(wid, i).reshape(-1) for i in range(len(mats_def))]
        samples[wid] = [x[:CPU_SAMPLE] for x in xs]
        n = sum(x.size for x in xs)
        ws = [torch.from_numpy(x.view(np.int16)).to(dev) for x in xs]
        cms = codec.compress_block(ws, cap=CAP)
        outs = [torch.empty(x.size, dtype=torch.bfloat16, device=dev) for x in xs]
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        abis, ptrs = [m.abi() for m in cms], [o.data_ptr() for o in outs]
        stream = torch.cuda.current_stream(dev)
        sh = int(stream.cuda_stream)

        def step():
            df11.check(df11.df11_decode_block_batch(abis, ptrs, status.data_ptr(), sh),
                       "df11_decode_block_batch")

        for _ in range(max(3, warmup)):
            step()
        torch.cuda.synchronize()
        exact = int(status.item()) == 0 and all(
            torch.equal(o.view(torch.int16), w) for o, w in zip(outs, ws))
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        for i, (a, b) in enumerate(evs):
            flush.fill_(i & 0xFF)
            a.record(stream)
            step()
            b.record(stream)
        torch.cuda.synchronize()
        ms = statistics.median(a.elapsed_time(b) for a, b in evs)
        algo = sum(m.read_bytes + m.index_bytes for m in cms) + 2 * n
        lines[workloads.workload_name(wid)] = {
            "weights": n, "matrices": len(xs), "ms_per_launch": ms,
            "value": 2 * n / (ms / 1e3) / 1e9, "unit": "GB/s", "weights_per_s": n / (ms / 1e3),
            "ratio": sum(m.stored_bytes for m in cms) / (2 * n), "bit_exact": exact,
            "max_code_len": max(int(m.codebook.max_len) for m in cms),
            "l2": f"{L2_FLUSH_BYTES >> 20} MiB written before each timed launch",
            "roofline": {"bound": "hbm", "achieved": algo / (ms / 1e3) / 1e9, "peak": peak,
                         "unit": "GB/s", "frac": algo / (ms / 1e3) / 1e9 / peak,
                         "peak_kind": peak_kind, "algorithmic_bytes_per_launch": algo}}
        del cms, outs, ws
        torch.cuda.empty_cache()
    del flush
    return lines, samples


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    wid = args.workload
    name = workloads.workload_name(wid)
    mats = workloads.WORKLOADS[wid][1]
    # each step: the oracle decodes the smallest matrix of the workload
    idx = min(range(len(mats)), key=lambda i: int(np.prod(mats[i][1])))
    x = workloads.matrix(wid, idx).reshape(-1)
    enc = oracle.encode(x, cap=CAP)
    for _ in range(args.warmup):
        oracle.decode(enc)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        out = oracle.decode(enc)
    dt = time.perf_counter() - t0
    assert np.array_equal(out, x)
    gbs = 2 * x.size * args.steps / dt / 1e9
    sample = f"matrix {mats[idx][0]} {mats[idx][1][0]}x{mats[idx][1][1] if len(mats[idx][1]) > 1 else ''} ({x.size} weights) of {name} per step"
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u8",
        "data": "synthetic",
        "config": {"workload": name, "weights": int(x.size), "sample": sample},
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_df11(args):
    import torch
    rank, world, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        dist = None
    dev = torch.device("cuda", torch.cuda.current_device())
    import lossless_bf16_weight_df11_b200 as df11
    from lossless_bf16_weight_df11_b200 import build as df11_build
    if not os.path.exists(df11.library_path()):
        df11_build.build()
    import lossless_bf16_weight_df11_b200.codec as codec

    wid = args.workload
    name = workloads.workload_name(wid)
    mats_def = workloads.WORKLOADS[wid][1]
    xs = [workloads.matrix(wid, i) for i in range(len(mats_def))]
    n_total = sum(x.size for x in xs)

    # compress on the GPU (histogram -> codebook -> encode), and time it after
    # a small warm-up compression (first launches load the kernels)
    ws = [torch.from_numpy(x.reshape(-1).view(np.int16)).to(dev) for x in xs]
    codec.compress(ws[0][:65536], cap=CAP)
    torch.cuda.synchronize()
    comp_t0 = time.perf_counter()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    cms = [codec.compress(w, cap=CAP) for w in ws]
    ev1.record()
    torch.cuda.synchronize()
    compress_ms = ev0.elapsed_time(ev1)
    compress_wall = time.perf_counter() - comp_t0
    # the batched compressor (two host round trips for the whole block)
    codec.compress_block([ws[0][:65536], ws[1][:65536]], cap=CAP)
    torch.cuda.synchronize()
    eb0, eb1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    eb0.record()
    cms_b = codec.compress_block(ws, cap=CAP)
    eb1.record()
    torch.cuda.synchronize()
    compress_block_ms = eb0.elapsed_time(eb1)
    same = all(int(a.total_bits) == int(b.total_bits) and torch.equal(a.stream, b.stream)
               for a, b in zip(cms, cms_b))
    del cms_b
    # the all-device compressor (codebooks built by a kernel)
    codec.compress_block_device([ws[0][:65536], ws[1][:65536]], cap=CAP)
    torch.cuda.synchronize()
    ed0, ed1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ed0.record()
    cms_d = codec.compress_block_device(ws, cap=CAP)
    ed1.record()
    torch.cuda.synchronize()
    compress_device_ms = ed0.elapsed_time(ed1)
    same_device = all(int(a.total_bits) == int(b.total_bits) and torch.equal(a.stream, b.stream)
                      and torch.equal(a.tables, b.tables) for a, b in zip(cms, cms_d))
    del cms_d
    read_bytes = sum(m.read_bytes for m in cms)
    index_bytes = sum(m.index_bytes for m in cms)
    seg_read = sum(m.seg_read_bytes for m in cms)
    seg_index_bytes = sum(4 * (-(-m.n // df11.SEGMENT) + 1) for m in cms)
    stored = sum(m.stored_bytes for m in cms)
    ratio = stored / (2 * n_total)
    # the indexed decoder's bytes: the format's arrays and the run index read,
    # the BF16 written
    algo_bytes = read_bytes + index_bytes + 2 * n_total

    outs = [torch.empty(x.shape, dtype=torch.bfloat16, device=dev) for x in xs]
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    abis = [m.abi() for m in cms]
    out_ptrs = [o.data_ptr() for o in outs]
    sh = int(stream.cuda_stream)

    def step():
        st = df11.df11_decode_block_batch(abis, out_ptrs, status.data_ptr(), sh)
        if st:
            raise df11.DF11Error(st, "df11_decode_block_batch")

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise df11.DF11Error(int(status.item()), "decode (device)")
    bit_exact = None
    if not args.no_verify:
        bit_exact = all(torch.equal(o.reshape(-1).view(torch.int16), w) for o, w in zip(outs, ws))
        if not bit_exact:
            raise SystemExit("decode is not bit-exact")

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        with torch.cuda.stream(stream):
            t_start.record(stream)
            for i in range(args.steps):
                starts[i].record(stream)
                step()
                ends[i].record(stream)
            t_end.record(stream)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    total_ms = max_over_ranks(t_start.elapsed_time(t_end), dist, dev)
    per_launch_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    ms_per_step = total_ms / args.steps
    value = 2 * n_total * world * args.steps / (total_ms / 1e3) / 1e9
    if int(status.item()) != 0:
        raise df11.DF11Error(int(status.item()), "decode (device)")

    # ---- the same block through the two other decoders: with the segment
    # index (each lane decodes 64 codes from a known bit) and with no index
    # (per-unit prefix sums of the threads' counts); and the time to build
    # each index (once, when a matrix is placed on the device)
    other = None
    if args.cap32:
        other = {}
        for dec_name, kw, kern, algo in (
                ("seg_index", (False, True), "decode_seg_kernel", seg_read + 2 * n_total),
                ("no_index", (False, False), "decode_kernel", read_bytes + 2 * n_total)):
            abis_o = [m.abi(*kw) for m in cms]

            def step_o():
                st = df11.df11_decode_block_batch(abis_o, out_ptrs, status.data_ptr(), sh)
                if st:
                    raise df11.DF11Error(st, "df11_decode_block_batch")

            for o in outs:
                o.zero_()
            with torch.cuda.stream(stream):
                for _ in range(args.warmup):
                    step_o()
            torch.cuda.synchronize()
            ok_o = int(status.item()) == 0 and all(
                torch.equal(o.reshape(-1).view(torch.int16), w) for o, w in zip(outs, ws))
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                e0.record(stream)
                for _ in range(args.steps):
                    step_o()
                e1.record(stream)
            torch.cuda.synchronize()
            ms_o = e0.elapsed_time(e1) / args.steps
            other[dec_name] = {"ms_per_step": ms_o, "value": 2 * n_total / (ms_o / 1e3) / 1e9,
                           "unit": "GB/s", "kernel": kern, "algorithmic_bytes_per_launch": algo,
                           "roofline_frac": algo / (ms_o / 1e3) / 1e9 / measured_peak()[0],
                           "bit_exact": ok_o}
        ri_status = torch.zeros(1, dtype=torch.int32, device=dev)
        tmp_ri = [torch.empty_like(m.run_index) for m in cms]
        tmp_si = [torch.empty_like(m.seg_index) for m in cms]

        def build_run_index():
            for m, r in zip(cms, tmp_ri):
                df11.check(df11.df11_build_run_index(m.abi(False, False), r.data_ptr(),
                                                     ri_status.data_ptr(), sh), "df11_build_run_index")

        def build_seg_index():
            for m, r in zip(cms, tmp_si):
                df11.check(df11.df11_build_segment_index(m.abi(False, False), r.data_ptr(),
                                                         ri_status.data_ptr(), sh),
                           "df11_build_segment_index")

        build_ms = {}
        for nm, fn in (("run_index", build_run_index), ("seg_index", build_seg_index)):
            with torch.cuda.stream(stream):
                fn()
                b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                b0.record(stream)
                fn()
                b1.record(stream)
            torch.cuda.synchronize()
            build_ms[nm] = b0.elapsed_time(b1)
        # (entries past the segment index's last one are padding, never written)
        same_index = (all(torch.equal(a, m.run_index) for a, m in zip(tmp_ri, cms)) and
                      all(torch.equal(a[:-(-m.n // df11.SEGMENT) + 1], m.seg_index[:-(-m.n // df11.SEGMENT) + 1])
                          for a, m in zip(tmp_si, cms)))
        del tmp_ri, tmp_si
        other["index_build"] = {"run_index_ms": build_ms["run_index"],
                                "seg_index_ms": build_ms["seg_index"],
                                "run_index_bytes": index_bytes, "seg_index_bytes": seg_index_bytes,
                                "rebuilt_identical": same_index and int(ri_status.item()) == 0}

    # ---- the rANS variant of the exponent coding on the same block: its
    # ratio and decode time beside the Huffman format's, launches alternated
    rans_line = None
    if args.rans_steps > 0:
        peak_r, peak_kind_r = measured_peak()
        rans_line = time_rans(torch, df11, ws, outs, out_ptrs, status, dev, args.rans_steps,
                              args.warmup, peak_r, peak_kind_r, n_total, ratio, step, stream)

    # ---- end to end through the C ABI with host buffers (pinned)
    e2e = None
    if args.e2e_steps > 0:
        e2e = end_to_end(torch, df11, codec, cms, xs, dev, args.e2e_steps, dist, world)

    # ---- the same block coded under the format's 32-bit cap (codes longer
    # than the decode table take the length search): reported beside
    cap32 = None
    if args.cap32:
        cms32 = [codec.compress(w, cap=32) for w in ws]
        abis32 = [m.abi() for m in cms32]
        algo32 = sum(m.read_bytes + m.index_bytes for m in cms32) + 2 * n_total

        def step32():
            st = df11.df11_decode_block_batch(abis32, out_ptrs, status.data_ptr(), sh)
            if st:
                raise df11.DF11Error(st, "df11_decode_block_batch")

        with torch.cuda.stream(stream):
            for _ in range(args.warmup):
                step32()
        torch.cuda.synchronize()
        ok32 = all(torch.equal(o.reshape(-1).view(torch.int16), w) for o, w in zip(outs, ws))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(args.steps):
                step32()
            e1.record(stream)
        torch.cuda.synchronize()
        ms32 = e0.elapsed_time(e1) / args.steps
        cap32 = {"ms_per_step": ms32, "value": 2 * n_total / (ms32 / 1e3) / 1e9, "unit": "GB/s",
                 "ratio": sum(m.stored_bytes for m in cms32) / (2 * n_total),
                 "roofline_achieved": algo32 / (ms32 / 1e3) / 1e9, "bit_exact": ok32,
                 "max_code_len": max(int(m.codebook.max_len) for m in cms32)}
        del cms32, abis32

    peak, peak_kind = measured_peak()
    # ---- the encode path on the device alone (S2 histogram + S4 encode):
    # the kernels of the 7 matrices back to back, codebooks already built,
    # rewriting the same compressed buffers with the same bytes
    encode = None
    if args.encode_steps > 0:
        encode = time_encode(torch, df11, cms, ws, dev, args.encode_steps, peak, peak_kind)
    # ---- fused decode -> matmul (y = x W^T, W never materialised) beside
    # decode followed by a cuBLAS matmul, and the matmul alone on resident
    # BF16 weights
    # ---- a whole transformer block held in DF11 form: decode (one launch)
    # then the block's forward, beside the same forward on resident weights
    blockfw = None
    if args.block_steps > 0 and wid in BLOCK_SHAPES:
        blockfw = time_block_forward(torch, cms, ws, mats_def, wid, dev, args.block_steps)
    fused = None
    tc_gemm = None
    if args.matmul_steps > 0:
        fused = [time_fused_matmul(torch, df11, cms, abis, outs, out_ptrs, status, xs_shapes(mats_def),
                                   dev, b, args.matmul_steps, peak, peak_kind) for b in (1, 8)]
        tf, tf_kind = measured_tensor_peak()
        tc_gemm = []
        for b in (16, 64, 256, 1024, 2048):
            tc_gemm.append(time_tc_gemm(torch, df11, cms, out_ptrs, outs, status, xs_shapes(mats_def),
                                        dev, b, args.matmul_steps, tf, tf_kind, peak))
            torch.cuda.empty_cache()

    configs, cpu_plan = None, None
    if args.config_steps > 0:
        peak_c, peak_kind_c = measured_peak()
        configs, samples = time_configs(torch, df11, codec, dev, args.config_steps, args.warmup,
                                        peak_c, peak_kind_c, wid, xs)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            cpu_plan = cpu_baseline_plan(samples)
        del samples

    avg_launch_ms = statistics.mean(per_launch_ms)
    achieved = algo_bytes / (avg_launch_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": profiled_traffic(name),
                "peak_kind": peak_kind, "kernel": "decode_idx_kernel",
                "algorithmic_bytes_per_launch": algo_bytes,
                "run_index_bytes_per_launch": index_bytes,
                "frac_of_8TBps": achieved / 8000.0,
                "median_launch_ms": statistics.median(per_launch_ms)}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sample = [xs[i] for i, (nm, _) in enumerate(mats_def) if nm in ORACLE_SAMPLE] or xs[:1]
        gbs, dt, ns = oracle_decode_rate(sample, ORACLE_SAMPLE)
        cpu = {"value": gbs, "unit": "GB/s", "cores": 1, "kind": "oracle", **cpu_info(),
               "sample": f"{'+'.join(nm for nm, _ in mats_def if nm in ORACLE_SAMPLE) or 'first matrix'}"
                         f" of {name}: {ns} weights decoded bit-serially in {dt:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "u8", "data": "synthetic",
            "config": {"workload": name, "matrices": len(xs), "weights_per_gpu": int(n_total),
                       "codebooks": len(xs), "l2": "inputs (2.9 GB) larger than L2; no flush",
                       "parallelism": f"replica per GPU x{world}"},
            "weights_per_s": n_total * world * args.steps / (total_ms / 1e3),
            "ratio": ratio, "bits_per_weight": 16 * ratio, "bit_exact": bit_exact,
            "compress": {"ms": compress_ms, "wall_s": compress_wall,
                         "input_GBps": 2 * n_total / (compress_ms / 1e3) / 1e9,
                         "includes": "per matrix: histogram, its copy to the host, the host "
                                     "codebook and tables, encode"},
            "compress_block": {"ms": compress_block_ms,
                               "input_GBps": 2 * n_total / (compress_block_ms / 1e3) / 1e9,
                               "same_as_per_matrix": same,
                               "includes": "all histograms, one copy to the host, host codebooks "
                                           "and tables, all encodes, one copy of the status words"},
            "compress_block_device": {"ms": compress_device_ms,
                                      "input_GBps": 2 * n_total / (compress_device_ms / 1e3) / 1e9,
                                      "same_as_per_matrix": same_device,
                                      "includes": "all histograms, codebooks and tables built on the "
                                                  "device, one copy of codebooks and sizes to the "
                                                  "host, all encodes, one copy of the status words"},
            "encode": encode,
            "fused_matmul": fused,
            "tc_gemm": tc_gemm,
            "block_forward": blockfw,
            "rans": rans_line,
            "code_len_cap": CAP,
            "max_code_len": max(int(m.codebook.max_len) for m in cms),
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "cap32": cap32,
            "configs": configs, "cpu_baseline_plan": cpu_plan, "other_decoders": other,
            "gpu_launches": args.steps, "clocks": clk.summary(),
        }
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def time_rans(torch, df11, ws, outs, out_ptrs, status, dev, steps, warmup, peak, peak_kind,
              n_total, huffman_ratio, huffman_step, huffman_stream):
    """The block coded with the rANS variant (df11_rans.h): compression on the
    device, then `steps` decode launches (all matrices in one launch), each
    followed by one launch of the Huffman format's decode (huffman_step, on
    huffman_stream), every launch timed with CUDA events on its stream, after
    `warmup` untimed ones and a bit-exactness check.  Alternating the two
    gives both the same clocks and the same L2 history."""
    import lossless_bf16_weight_df11_b200.rans as rans
    rans.compress_block([ws[0][:65536]])
    torch.cuda.synchronize()
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record()
    rms = rans.compress_block(ws)
    c1.record()
    torch.cuda.synchronize()
    abis = [m.abi() for m in rms]
    stream = torch.cuda.Stream(device=dev)
    sh = int(stream.cuda_stream)
    status.zero_()

    def step():
        st = df11.df11_rans_decode_batch(abis, out_ptrs, status.data_ptr(), sh)
        if st:
            raise df11.DF11Error(st, "df11_rans_decode_batch")

    with torch.cuda.stream(stream):
        for _ in range(max(1, warmup)):
            step()
    torch.cuda.synchronize()
    ok = int(status.item()) == 0 and all(
        torch.equal(o.reshape(-1).view(torch.int16), w) for o, w in zip(outs, ws))
    def pair():
        return torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    evs = [pair() for _ in range(steps)]
    evh = [pair() for _ in range(steps)]
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        for (a, b), (c, d) in zip(evs, evh):
            with torch.cuda.stream(stream):
                a.record(stream)
                step()
                b.record(stream)
            stream.synchronize()
            with torch.cuda.stream(huffman_stream):
                c.record(huffman_stream)
                huffman_step()
                d.record(huffman_stream)
            torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise df11.DF11Error(int(status.item()), "decode (device)")
    t = [a.elapsed_time(b) for a, b in evs]
    th = [c.elapsed_time(d) for c, d in evh]
    avg = statistics.mean(t)
    algo = sum(m.read_bytes for m in rms) + 2 * n_total
    r = sum(m.stored_bytes for m in rms) / (2 * n_total)
    out = {"ratio": r, "bits_per_weight": 16 * r, "bit_exact": ok, "launches": steps,
           "ms_per_launch": avg, "median_ms": statistics.median(t),
           "value": 2 * n_total / (avg / 1e3) / 1e9, "unit": "GB/s",
           "compress_block_ms": c0.elapsed_time(c1),
           "roofline": {"bound": "hbm", "achieved": algo / (avg / 1e3) / 1e9, "peak": peak,
                        "unit": "GB/s", "frac": algo / (avg / 1e3) / 1e9 / peak,
                        "peak_kind": peak_kind, "kernel": "rans_decode_kernel",
                        "algorithmic_bytes_per_launch": algo},
           "vs_huffman": {"stored_size": r / huffman_ratio,
                          "huffman_median_ms_alternated": statistics.median(th),
                          "decode_time": statistics.median(t) / statistics.median(th)},
           "clocks": clk.summary()}
    del rms
    return out


def time_encode(torch, df11, cms, ws, dev, steps, peak, peak_kind):
    """Device time of df11_histogram + df11_encode over the block's matrices
    (6 kernel launches per matrix), averaged over `steps` passes after one
    warm-up pass."""
    stream = torch.cuda.Stream(device=dev)
    sh = int(stream.cuda_stream)
    hist = torch.empty(256, dtype=torch.int64, device=dev)
    wsb = torch.empty(max(16, max(int(m.sizes.workspace_bytes) for m in cms)), dtype=torch.uint8,
                      device=dev)
    status = torch.zeros(2, dtype=torch.int32, device=dev)
    outs = [df11.df11_encoded(stream=m.stream.data_ptr(), gaps=m.gaps.data_ptr(),
                              block_pos=m.block_pos.data_ptr(),
                              sign_mantissa=m.sign_mantissa.data_ptr(),
                              block_max=status.data_ptr() + 4) for m in cms]

    def one_pass():
        for m, w, o in zip(cms, ws, outs):
            n = w.numel()
            df11.check(df11.df11_histogram(w.data_ptr(), n, hist.data_ptr(), sh), "df11_histogram")
            df11.check(df11.df11_encode(w.data_ptr(), n, m.codebook, m.total_bits, o, wsb.data_ptr(),
                                        wsb.numel(), status.data_ptr(), sh), "df11_encode")

    one_pass()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        one_pass()
    e1.record(stream)
    torch.cuda.synchronize()
    if int(status[0].item()) != 0:
        raise df11.DF11Error(int(status[0].item()), "encode (device)")
    ms = e0.elapsed_time(e1) / steps
    n_total = sum(w.numel() for w in ws)
    algo = 2 * n_total + sum(int(m.stored_bytes) for m in cms)  # input read once + output written
    return {"ms": ms, "input_GBps": 2 * n_total / (ms / 1e3) / 1e9, "launches": 6 * len(cms),
            "roofline": {"bound": "hbm", "achieved": algo / (ms / 1e3) / 1e9, "peak": peak,
                         "unit": "GB/s", "frac": algo / (ms / 1e3) / 1e9 / peak,
                         "peak_kind": peak_kind, "algorithmic_bytes": algo},
            "note": "histogram + encode kernels back to back, codebooks built beforehand"}


# (hidden, heads, kv_heads, ffn) of the block workloads
BLOCK_SHAPES = {3: (4096, 32, 8, 14336), 5: (8192, 64, 8, 28672)}


def time_block_forward(torch, cms, ws, mats_def, wid, dev, steps):
    """DF11Block.forward (decode of the seven matrices + the block) against the
    same forward on the resident BF16 weights, for 16 and 2048 tokens."""
    import dataclasses
    import lossless_bf16_weight_df11_b200.block as blockmod
    shape = blockmod.BlockShape(*BLOCK_SHAPES[wid])
    names = [nm for nm, _ in mats_def]
    mats = {nm: dataclasses.replace(m, shape=tuple(sh)) for nm, m, (_, sh) in zip(names, cms, mats_def)}
    wts = {nm: w.view(torch.bfloat16).reshape(sh) for nm, w, (_, sh) in zip(names, ws, mats_def)}
    blk = blockmod.DF11Block(mats, shape)
    g = torch.Generator(device=dev)
    g.manual_seed(77)
    out = []
    for tokens in (16, 2048):
        x = torch.randn(1, tokens, shape.hidden, generator=g, device=dev).to(torch.bfloat16)

        def timed(fn):
            for _ in range(2):
                fn()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(steps):
                fn()
            e1.record()
            torch.cuda.synchronize()
            return e0.elapsed_time(e1) / steps

        same = bool(torch.equal(blk.forward(x), blk.forward_reference(x, wts)))
        t_df11 = timed(lambda: blk.forward(x))
        t_ref = timed(lambda: blk.forward_reference(x, wts))
        out.append({"tokens": tokens, "df11_ms": t_df11, "bf16_resident_ms": t_ref,
                    "decode_overhead_ms": t_df11 - t_ref, "bit_identical": same})
    return out


def xs_shapes(mats_def):
    return [tuple(shape) for _, shape in mats_def]


def time_fused_matmul(torch, df11, cms, abis, outs, out_ptrs, status, shapes, dev, batch, steps,
                      peak, peak_kind):
    """Per step, for all matrices W_i (rows x cols) of the block and BF16
    activations x_i (batch x cols): y_i += x_i W_i^T.  Three ways: the fused
    kernel (one launch); decode into BF16 then torch.matmul (cuBLAS); the
    matmul alone with the BF16 weights already resident."""
    g = torch.Generator(device=dev)
    g.manual_seed(1234 + batch)
    xs = [torch.randn(batch, c, generator=g, device=dev).to(torch.bfloat16) for _, c in shapes]
    ys = [torch.zeros(batch, r, dtype=torch.float32, device=dev) for r, _ in shapes]
    ios = [df11.df11_matmul_io(rows=r, cols=c, x=x.data_ptr(), y=y.data_ptr())
           for (r, c), x, y in zip(shapes, xs, ys)]
    stream = torch.cuda.current_stream(dev)
    sh = int(stream.cuda_stream)
    ws_bf16 = [o.view(r, c) for o, (r, c) in zip(outs, shapes)]

    def fused():
        df11.check(df11.df11_decode_matmul_batch(abis, ios, batch, status.data_ptr(), sh),
                   "df11_decode_matmul_batch")

    def decode_then_matmul():
        df11.check(df11.df11_decode_block_batch(abis, out_ptrs, status.data_ptr(), sh),
                   "df11_decode_block_batch")
        for x, w, y in zip(xs, ws_bf16, ys):
            y.add_(torch.matmul(x, w.t()).float())

    def matmul_only():
        for x, w, y in zip(xs, ws_bf16, ys):
            y.add_(torch.matmul(x, w.t()).float())

    def timed(fn):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    t_fused = timed(fused)
    # agreement with the unfused path on one step (FP32 sums in another order)
    for y in ys:
        y.zero_()
    fused()
    ref = [torch.matmul(x.double(), w.double().t()) for x, w in zip(xs, ws_bf16)]
    bound_ok = all(bool(((y.double() - r).abs() <= (x.double().abs() @ w.double().abs().t())
                         * (w.shape[1] + 8) * 2.0 ** -24 * 1.01).all())
                   for x, w, y, r in zip(xs, ws_bf16, ys, ref))
    del ref
    t_unfused = timed(decode_then_matmul)
    t_mm = timed(matmul_only)
    if int(status.item()) != 0:
        raise df11.DF11Error(int(status.item()), "fused matmul (device)")
    algo = (sum(m.read_bytes for m in cms) + sum(2 * x.numel() for x in xs)
            + sum(8 * y.numel() for y in ys))  # compressed W, x, y read and written
    return {"batch": batch, "fused_ms": t_fused, "decode_then_matmul_ms": t_unfused,
            "matmul_only_ms": t_mm, "speedup_vs_decode_then_matmul": t_unfused / t_fused,
            "within_fp32_sum_bound": bound_ok,
            "roofline": {"bound": "hbm", "achieved": algo / (t_fused / 1e3) / 1e9, "peak": peak,
                         "unit": "GB/s", "frac": algo / (t_fused / 1e3) / 1e9 / peak,
                         "peak_kind": peak_kind, "algorithmic_bytes": algo}}


def time_tc_gemm(torch, df11, cms, out_ptrs, outs, status, shapes, dev, batch, steps, peak_tf,
                 peak_tf_kind, hbm_peak):
    """Per step, for all matrices W_i (rows x cols) of the block and BF16
    activations x_i (batch x cols): y_i += x_i W_i^T.  Three ways: the
    tensor-core fused kernel (df11_decode_gemm_batch: W decoded into the MMA's
    operand tiles, one pass per 256 activation rows); decode into BF16 then
    torch.matmul (cuBLAS); the matmul alone with the BF16 weights resident."""
    g = torch.Generator(device=dev)
    g.manual_seed(4321 + batch)
    xs = [torch.randn(batch, c, generator=g, device=dev).to(torch.bfloat16) for _, c in shapes]
    ys = [torch.zeros(batch, r, dtype=torch.float32, device=dev) for r, _ in shapes]
    ios = [df11.df11_matmul_io(rows=r, cols=c, x=x.data_ptr(), y=y.data_ptr())
           for (r, c), x, y in zip(shapes, xs, ys)]
    abis = [m.abi() for m in cms]
    stream = torch.cuda.current_stream(dev)
    sh = int(stream.cuda_stream)
    ws_bf16 = [o.view(r, c) for o, (r, c) in zip(outs, shapes)]

    def fused():
        df11.check(df11.df11_decode_gemm_batch(abis, ios, batch, status.data_ptr(), sh),
                   "df11_decode_gemm_batch")

    def decode_then_matmul():
        df11.check(df11.df11_decode_block_batch(abis, out_ptrs, status.data_ptr(), sh),
                   "df11_decode_block_batch")
        for x, w, y in zip(xs, ws_bf16, ys):
            y.add_(torch.matmul(x, w.t()).float())

    def matmul_only():
        for x, w, y in zip(xs, ws_bf16, ys):
            y.add_(torch.matmul(x, w.t()).float())

    def timed(fn):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    t_fused = timed(fused)
    # one step from zero, checked on 16 sampled rows of every W against a
    # float64 product, within (cols + 8) ulps of the sum of |w x|
    for y in ys:
        y.zero_()
    fused()
    decode_then_matmul()  # fills the BF16 weights (and adds the cuBLAS product to y)
    for y in ys:
        y.zero_()
    fused()
    ok = int(status.item()) == 0
    for x, w, y in zip(xs, ws_bf16, ys):
        rows = torch.randperm(w.shape[0], generator=torch.Generator().manual_seed(batch))[:16].to(dev)
        wr = w[rows].double()
        ref = x.double() @ wr.t()
        bound = (x.double().abs() @ wr.abs().t()) * (w.shape[1] + 8) * 2.0 ** -23 * 1.01
        ok = ok and bool(((y[:, rows].double() - ref).abs() <= bound).all())
    t_unfused = timed(decode_then_matmul)
    t_mm = timed(matmul_only)
    if int(status.item()) != 0:
        raise df11.DF11Error(int(status.item()), "tensor-core fused GEMM (device)")
    flops = 2.0 * batch * sum(r * c for r, c in shapes)
    passes = -(-batch // df11.GEMM_MAX_BATCH)
    algo = (passes * sum(m.seg_read_bytes for m in cms) + sum(2 * x.numel() for x in xs)
            + sum(8 * y.numel() for y in ys))  # compressed W per pass, x, y read and written
    return {"batch": batch, "fused_ms": t_fused, "decode_then_matmul_ms": t_unfused,
            "matmul_only_ms": t_mm, "speedup_vs_decode_then_matmul": t_unfused / t_fused,
            "passes": passes, "within_fp32_bound_sampled": ok, "kernel": "decode_gemm_tc_kernel",
            "roofline": {"bound": "tensor", "achieved": flops / (t_fused / 1e3) / 1e12,
                         "peak": peak_tf, "unit": "TFLOP/s",
                         "frac": flops / (t_fused / 1e3) / 1e12 / peak_tf, "peak_kind": peak_tf_kind,
                         "flops": flops},
            "hbm_view": {"achieved": algo / (t_fused / 1e3) / 1e9, "peak": hbm_peak, "unit": "GB/s",
                         "frac": algo / (t_fused / 1e3) / 1e9 / hbm_peak, "bytes": algo}}


def end_to_end(torch, df11, codec, cms, xs, dev, steps, dist, world):
    """Host-resident compressed block -> host BF16 through the library's
    pipelined host-buffer call (df11_decode_host_batch): per piece of a
    matrix (256 blocks, doubling up to 4096), its stored arrays are copied in from
    page-locked memory, its run index is built, it is decoded and its BF16
    words are copied out, both copy directions and the kernels overlapping
    from piece to piece.  Every step, all timed."""
    hms = [codec.HostMatrix.from_matrix(m) for m in cms]
    abis = [h.abi() for h in hms]
    scratch = codec.host_scratch(hms, dev)
    n_total = sum(x.size for x in xs)
    host_out = [torch.empty(x.shape, dtype=torch.bfloat16, pin_memory=True) for x in xs]
    ptrs = [o.data_ptr() for o in host_out]
    h2d = sum(h.h2d_bytes for h in hms)  # + 21 bytes re-read at each cut between pieces
    d2h = 2 * n_total
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    sh = int(stream.cuda_stream)

    def step():
        st = df11.df11_decode_host_batch(abis, ptrs, scratch.data_ptr(), scratch.numel(),
                                         status.data_ptr(), sh)
        if st:
            raise df11.DF11Error(st, "df11_decode_host_batch")

    for _ in range(2):
        step()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1), dist, dev)
    ok = all(torch.equal(h.view(torch.int16).reshape(-1), torch.from_numpy(x.reshape(-1).view(np.int16)))
             for h, x in zip(host_out, xs))
    if int(status.item()) != 0 or not ok:
        raise SystemExit("end-to-end decode is not bit-exact")
    return {"value": 2 * n_total * world * steps / (ms / 1e3) / 1e9, "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": ms / steps, "call": "df11_decode_host_batch",
            "host_memory": "page-locked", "scratch_bytes": int(scratch.numel())}


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_df11(args)


if __name__ == "__main__":
    sys.exit(main())
