#!/usr/bin/env python
"""Benchmark of the CacheGen KV-cache codec (libcachegen) on B200.

One step = one pass of the whole hot path over the Llama-2-7B-shaped MHA cache
(32 layers x K/V x 32 kv_heads x 128 head_dim, fp16, 10,752 tokens = 7 chunks
of 1,536; seeded AR(1) walks with 1% x8 outlier channels, seed 2; balanced
level): cg_encode of all 7 chunks, then cg_decode_into of all 7 containers into
one contiguous KV buffer.  Inputs (5.6 GB) are resident in HBM and larger than
L2, so no flush is needed between iterations.

Prints one JSON line.  `value` is the round-trip throughput (fp16 bytes per
step / step time, GB/s); encode and decode are also reported on their own,
with their fraction of the HBM roofline and the compression ratio.
`--impl reference` times the plain CPU oracle instead (the only comparison
arm this project has), on a bounded sample of the same workload.
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
from pathlib import Path

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

WORKLOAD = dict(name="llama2_7b", L=32, H=32, D=128, T=10752, C=1536, seed=2, rho=0.95,
                p_out=0.01, m_out=8.0, level=1)
METRIC = "cg_decode / cg_encode GB/s (fp16 KV) on 1 B200, % of HBM roofline, compression ratio"
FALLBACK_HBM_GBS = 6650.0
# DRAM bytes (read + write) per fp16 value of decode_kernel from one ncu capture
# of the current kernel on a Llama-2-7B-shaped case (32x2x3072x32x128 =
# 805,306,368 values: 352.9 MB read + 1,557.3 MB written); the bench reports it
# scaled by its own value count.  The capture ends with up to one L2 (126 MB)
# of written lines not yet in DRAM, so this slightly undercounts.
DECODE_DRAM_BYTES_PER_VALUE = (352_920_064 + 1_557_323_000) / 805_306_368
# Shared-memory wavefronts per warp-symbol of decode_kernel from the same
# capture (189,563,275 wavefronts for 805,306,368 symbols): the random slot-table
# lookups of 32 streams cost about four, the word refills, the code stores and
# loads and the table fills the rest.  An SM serves one wavefront per clock.
DECODE_SMEM_WAVEFRONTS_PER_WARP_SYMBOL = 189_563_275 / (805_306_368 / 32)


def smem_ceiling(symbols: int, ms: float, sm_mhz, sms: int):
    """The decode kernel against its shared-memory ceiling (one wavefront per
    SM per clock at the SM clock sampled during the timed region)."""
    if not sm_mhz or not ms or not sms:
        return None
    achieved = symbols / 32 * DECODE_SMEM_WAVEFRONTS_PER_WARP_SYMBOL / (ms * 1e-3)
    peak = sms * float(sm_mhz) * 1e6
    return {"bound": "smem", "achieved": round(achieved / 1e9, 1), "peak": round(peak / 1e9, 1),
            "unit": "G wavefronts/s", "frac": round(achieved / peak, 4),
            "wavefronts_per_warp_symbol": round(DECODE_SMEM_WAVEFRONTS_PER_WARP_SYMBOL, 2),
            "source": "ncu wavefronts per warp-symbol of a 3,072-token Llama-2-7B-shaped "
                      "capture; peak = SMs x sampled SM clock"}


def _peaks():
    try:
        return json.loads((ROOT / "MEASURED_PEAKS.json").read_text())
    except Exception:
        return {}


def _env_rank():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


def reduce_max(values, world, dist, device):
    """Max over ranks of each entry (the job's time is its slowest rank's);
    a no-op for one rank.  `device` is where the collective runs (the rank's
    GPU under NCCL, the CPU under gloo)."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_gbps(bytes_per_rank, world, ms):
    """Whole-job throughput: the bytes of all ranks over the max-over-ranks time."""
    return bytes_per_rank * world / ms / 1e6


def host_cores() -> int:
    """Cores this process may run on (the affinity mask, else the CPU count)."""
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def _oracle_sample(threads: int):
    """The CPU sample: one chunk of the workload cut into 16 independent 2-head
    slices ([32, 2, 1536, 2, 128] each, 50 MB of fp16), round-tripped through the
    oracle as max(16, threads) tasks (the slices in turn) on `threads` host
    threads, so that every core has work."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    from kv_cache_compression_cachegen_b200 import synth
    oracle.build()
    w = WORKLOAD
    slices = [synth.generate_cpu(w["L"], 2, w["D"], w["C"], seed=w["seed"] * 100 + i,
                                 rho=w["rho"], p_out=w["p_out"], m_out=w["m_out"])
              for i in range(16)]
    tasks = [slices[i % len(slices)] for i in range(max(16, threads))]

    def run_one(kv):
        rc, cont = oracle.encode_chunk(kv, 0, w["C"], w["level"])
        assert rc == 0
        rc, vals, n, _ = oracle.decode_chunk(cont, w["L"], 2, w["D"], w["C"], w["level"])
        assert rc == 0
        return cont.size

    nbytes = sum(s.nbytes for s in tasks)
    desc = (f"{len(tasks)} tasks over 16 slices of [{w['L']},2,{w['C']},2,{w['D']}] fp16 "
            f"(one {w['C']}-token chunk of the {w['name']} workload cut by head pairs), "
            f"{nbytes / 1e6:.0f} MB encode+decode")

    def step():
        t0 = time.perf_counter()
        with ThreadPoolExecutor(threads) as ex:
            sizes = list(ex.map(run_one, tasks))
        return time.perf_counter() - t0, sizes

    def one_core():
        """One slice on the calling thread: the oracle's single-core rate."""
        t0 = time.perf_counter()
        run_one(slices[0])
        return time.perf_counter() - t0, slices[0].nbytes

    step.one_core = one_core
    return step, nbytes, desc


def run_reference(args):
    rank, world, _ = _env_rank()
    if rank != 0:
        return 0
    threads = host_cores()
    step, nbytes, desc = _oracle_sample(threads)
    for _ in range(args.warmup):
        step()
    times = []
    for _ in range(args.steps):
        dt, _ = step()
        times.append(dt)
    total = sum(times)
    value = nbytes * args.steps / total / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * total / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "u8+f32", "data": "synthetic",
        "config": {"workload": WORKLOAD["name"], "sample": desc, "level": "balanced"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads,
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    import torch
    import torch.distributed as dist
    import kv_cache_compression_cachegen_b200 as cg
    from kv_cache_compression_cachegen_b200 import synth
    from kv_cache_compression_cachegen_b200 import torch_api as ta
    from kv_cache_compression_cachegen_b200.stats import clamp_counts

    rank, world, local = _env_rank()
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    cg.library()  # fails loudly if the native library is missing

    w = WORKLOAD
    L, H, D, T, C, level = w["L"], w["H"], w["D"], w["T"], w["C"], w["level"]
    nch = -(-T // C)
    shape = cg.Shape(L, H, D)
    stream = torch.cuda.Stream(dev)
    kv = torch.empty((L, 2, T, H, D), dtype=torch.int16, device=dev)
    synth.generate_gpu(kv, L, H, D, T, w["seed"] + 1000 * rank, w["rho"], w["p_out"],
                       w["m_out"], stream=stream)
    enc = ta.Encoder(shape, C, nch, dev)
    kv_out = torch.empty_like(kv)
    status = ta.new_status(dev)
    fp16_bytes = kv.numel() * 2

    nvtx = torch.cuda.nvtx

    def encode():
        nvtx.range_push("cg_encode")
        cg.check(cg.cg_encode(shape, kv, T, 0, nch, C, level, None, enc.out, enc.stride,
                              enc.sizes, enc.status, enc.workspace, enc.ws_bytes, stream))
        nvtx.range_pop()

    def decode():
        nvtx.range_push("cg_decode_into")
        cg.check(cg.cg_decode_into(shape, enc.out, enc.stride, nch, C, level, kv_out, T, status,
                                   stream))
        nvtx.range_pop()

    torch.cuda.synchronize(dev)
    for _ in range(max(args.warmup, 0)):
        encode()
        decode()
    torch.cuda.synchronize(dev)
    if ta.status_of(enc.status) != 0 or ta.status_of(status) != 0:
        raise RuntimeError(f"codec status {ta.status_of(enc.status)} / {ta.status_of(status)}")
    comp_bytes = int(enc.sizes.sum().item())

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    sampler = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.3)
    for i in range(args.steps):
        ev[i][0].record(stream)
        encode()
        ev[i][1].record(stream)
        decode()
        ev[i][2].record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    t_enc = [ev[i][0].elapsed_time(ev[i][1]) for i in range(args.steps)]
    t_dec = [ev[i][1].elapsed_time(ev[i][2]) for i in range(args.steps)]
    t_step = sum(t_enc) + sum(t_dec)
    t_step, te_sum, td_sum = reduce_max([t_step, sum(t_enc), sum(t_dec)], world, dist, dev)
    ms_step = t_step / args.steps
    ms_enc = te_sum / args.steps
    ms_dec = td_sum / args.steps
    peaks = _peaks()
    hbm = peaks.get("hbm_gbs", FALLBACK_HBM_GBS)
    peak_src = "measured" if "hbm_gbs" in peaks else "fallback"
    enc_gbps = fp16_bytes / ms_enc / 1e6
    dec_gbps = fp16_bytes / ms_dec / 1e6
    # algorithmic bytes: fp16 read + container write (encode); container read + fp16 write
    alg = fp16_bytes + comp_bytes
    enc_frac = alg / ms_enc / 1e6 / hbm
    dec_frac = alg / ms_dec / 1e6 / hbm
    # the target's own roofline definition: the same bytes over 8 TB/s
    enc_frac_8 = alg / ms_enc / 1e6 / 8000.0
    dec_frac_8 = alg / ms_dec / 1e6 / 8000.0
    clamped, deltas = clamp_counts(kv, kv_out, C, level)

    # ---- end to end through the C ABI with host buffers --------------------
    e2e = None
    if not args.skip_e2e:
        e2e = _e2e(args, torch, cg, ta, shape, kv, enc, kv_out, status, stream, dev, nch, C,
                   level, T, fp16_bytes, world, dist)
        full = _e2e(args, torch, cg, ta, shape, kv, enc, kv_out, status, stream, dev, nch, C,
                    level, T, fp16_bytes, world, dist, kv_back=True)
        e2e["with_decoded_kv_to_host"] = {
            "value": full["value"], "unit": full["unit"], "ms_per_step": full["ms_per_step"],
            "d2h_bytes_per_step": full["d2h_bytes_per_step"],
            "note": "the same step with every decoded chunk also copied back to pinned host "
                    "memory"}

    line = None
    if rank == 0:
        line = {
            "metric": METRIC,
            "value": round(job_gbps(fp16_bytes, world, ms_step), 2),
            "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "u8+f32", "data": "synthetic",
            "config": {"workload": f"{w['name']}: {L}x2x{H}x{D} fp16, {T} tokens = {nch} chunks "
                                   f"of {C}, balanced, AR(1) rho {w['rho']} with "
                                   f"{w['p_out']:.0%} x{w['m_out']:g} outliers, seed {w['seed']}",
                       "step": "cg_encode(7 chunks) + cg_decode_into(7 chunks)",
                       "l2": "inputs larger than L2 (5.6 GB), no flush",
                       "parallelism": f"dp{world} (independent caches per GPU)"},
            "encode_gbps": round(enc_gbps, 2), "decode_gbps": round(dec_gbps, 2),
            "encode_ms": round(ms_enc, 4), "decode_ms": round(ms_dec, 4),
            "encode_roofline_frac": round(enc_frac_8, 4),
            "decode_roofline_frac": round(dec_frac_8, 4),
            "roofline_frac_definition": "(fp16 bytes + container bytes) / 8 TB/s / time",
            "encode_frac_of_measured_hbm": round(enc_frac, 4),
            "decode_frac_of_measured_hbm": round(dec_frac, 4),
            "compression_ratio": round(fp16_bytes / comp_bytes, 4),
            "container_bytes": comp_bytes,
            "clamp_rate": clamped / deltas,
            "clamp_rate_def": "delta values whose code hit the [-127, 127] clamp (reconstruction "
                              "error above step/2 + half an fp16 spacing), over all delta values",
            "roofline": {"kernel": "decode_kernel (cg_decode_into)", "bound": "hbm",
                         "achieved": round(alg / ms_dec / 1e6, 1), "peak": hbm,
                         "peak_source": f"{peak_src} hbm_gbs", "unit": "GB/s",
                         "frac": round(dec_frac, 4),
                         "traffic": int(DECODE_DRAM_BYTES_PER_VALUE * (fp16_bytes // 2)),
                         "traffic_source": "ncu dram bytes per value of a 3,072-token "
                                           "Llama-2-7B-shaped capture, scaled by values",
                         "algorithmic_bytes": alg},
            # per step: quant, rans, offsets and compact for each half of the
            # chunks (cg_encode runs a call of two or more chunks as two
            # halves on two streams), then one decode
            "gpu_launches": ((8 if nch >= 2 else 4) + 1) * args.steps,
            "clocks": clocks,
        }
        # what bounds the decode kernel instead of HBM: its shared-memory wavefronts
        line["roofline"]["smem"] = smem_ceiling(
            fp16_bytes // 2, ms_dec, clocks.get("sm_mhz"),
            torch.cuda.get_device_properties(dev).multi_processor_count)
        if e2e is not None:
            line["e2e"] = e2e
        if not args.skip_cpu and world == 1:
            line["cpu_baseline"] = _cpu_baseline()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0


def _e2e(args, torch, cg, ta, shape, kv, enc, kv_out, status, stream, dev, nch, C, level, T,
         fp16_bytes, world, dist, kv_back=False):
    """Host in, host out, chunk by chunk: pinned fp16 KV -> H2D -> cg_encode ->
    D2H container (the sender's side), then H2D container -> cg_decode_into ->
    D2H status (the receiver's side; the decoded KV stays in device memory, where
    the model reads it).  Three streams overlap the copies of one chunk with the
    compute of another: `h2d` carries the fp16 chunks, `d2h` the containers out,
    `back` the containers in; `stream` runs the kernels.  kv_back=True also
    copies every decoded chunk back to pinned host memory (on `d2h`)."""
    L = shape.num_layers
    host_kv = torch.empty(kv.shape, dtype=kv.dtype, pin_memory=True)
    host_kv.copy_(kv)
    host_out = torch.empty(kv.shape, dtype=kv.dtype, pin_memory=True) if kv_back else None
    host_cont = torch.empty(enc.out.numel(), dtype=torch.uint8, pin_memory=True)
    host_status = torch.empty(2, dtype=torch.int32, pin_memory=True)
    sizes = enc.sizes.cpu().tolist()
    dev_cont = torch.empty_like(enc.out)
    h2d, d2h, back = (torch.cuda.Stream(dev) for _ in range(3))
    ev = lambda: torch.cuda.Event()  # noqa: E731
    kv_in, enc_done, out_done, in_done, dec_done = ([ev() for _ in range(nch)]
                                                    for _ in range(5))
    torch.cuda.synchronize(dev)
    steps = max(1, min(args.steps, 3))
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for s_ in (h2d, d2h, back):
        s_.wait_event(t0)
    for _ in range(steps):
        for k in range(nch):  # the fp16 chunks arrive back to back
            a, b = k * C, min(T, (k + 1) * C)
            with torch.cuda.stream(h2d):
                h2d.wait_event(enc_done[k])  # the previous step's encode of this chunk
                for l in range(L):
                    for kvi in range(2):
                        kv[l, kvi, a:b].copy_(host_kv[l, kvi, a:b], non_blocking=True)
                kv_in[k].record(h2d)
        for k in range(nch):
            o = k * enc.stride
            stream.wait_event(kv_in[k])
            cg.check(cg.cg_encode(shape, kv, T, k * C, 1, C, level, None, enc.out[o:],
                                  enc.stride, enc.sizes[k:], enc.status, enc.workspace,
                                  enc.ws_bytes, stream))
            enc_done[k].record(stream)
            with torch.cuda.stream(d2h):
                d2h.wait_event(enc_done[k])
                host_cont[o:o + sizes[k]].copy_(enc.out[o:o + sizes[k]], non_blocking=True)
                out_done[k].record(d2h)
            with torch.cuda.stream(back):
                back.wait_event(out_done[k])
                dev_cont[o:o + sizes[k]].copy_(host_cont[o:o + sizes[k]], non_blocking=True)
                in_done[k].record(back)
        for k in range(nch):
            o = k * enc.stride
            stream.wait_event(in_done[k])
            cg.check(cg.cg_decode_into(shape, dev_cont[o:], enc.stride, 1, C, level, kv_out, T,
                                       status, stream))
            if kv_back:
                dec_done[k].record(stream)
                a, b = k * C, min(T, (k + 1) * C)
                with torch.cuda.stream(d2h):
                    d2h.wait_event(dec_done[k])
                    for l in range(L):
                        for kvi in range(2):
                            host_out[l, kvi, a:b].copy_(kv_out[l, kvi, a:b], non_blocking=True)
        with torch.cuda.stream(stream):
            host_status[0:1].copy_(status, non_blocking=True)
            host_status[1:2].copy_(enc.status, non_blocking=True)
    for s_ in (h2d, d2h, back):
        stream.wait_stream(s_)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    if int(host_status[0]) != 0 or int(host_status[1]) != 0:
        raise RuntimeError(f"e2e status {host_status.tolist()}")
    if kv_back and not torch.equal(host_out[:, :, :C], kv_out[:, :, :C].cpu()):
        raise RuntimeError("e2e: decoded KV copied back differs from the device copy")
    ms = reduce_max([t0.elapsed_time(t1) / steps], world, dist, dev)[0]
    comp = sum(sizes)
    return {"value": round(job_gbps(fp16_bytes, world, ms), 3), "unit": "GB/s",
            "ms_per_step": round(ms, 3), "h2d_bytes_per_step": fp16_bytes + comp,
            "d2h_bytes_per_step": comp + 8 + (fp16_bytes if kv_back else 0),
            "overlap": "per-chunk copies on three streams"}


def _cpu_baseline():
    threads = host_cores()
    step, nbytes, desc = _oracle_sample(threads)
    dt, _ = step()
    dt1, nb1 = step.one_core()
    return {"value": round(nbytes / dt / 1e9, 4), "unit": "GB/s", "cores": threads,
            "kind": "oracle", "sample": desc,
            "single_core": {"value": round(nb1 / dt1 / 1e9, 4), "unit": "GB/s",
                            "sample": "the first of the 16 slices on one thread"}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--skip-cpu", action="store_true")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
