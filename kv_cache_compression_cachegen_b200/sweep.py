"""Throughput and compression ratio of the codec on the synthetic workloads
other than the bench's, one JSON line per measurement.

    python -m kv_cache_compression_cachegen_b200.sweep --config mistral7b
    python -m kv_cache_compression_cachegen_b200.sweep --config sweep
    python -m kv_cache_compression_cachegen_b200.sweep --config llama34b

mistral7b  the Mistral-7B shape (one 1,536-token chunk) at the three levels;
sweep      chunk sizes 512 / 1,024 / 1,536 / 2,048 x three levels x the two
           value distributions on the Mistral-7B shape at 32,768 tokens;
llama34b   the Llama-34B shape: first the three-level pre-encode of a
           13-chunk batch, as three cg_encode calls and as one
           cg_encode_levels call; then all 52 chunks pre-encoded at the three
           levels and decoded chunk by chunk with cg_decode_into following the
           per-chunk level schedule: once from device-resident containers
           (kernel-only) and once streamed from pinned host memory with the
           next chunk's host-to-device copy overlapping the current decode
           (end to end).

paged      the Llama-2-7B shape (balanced) decoded into a paged pool of
           16-token pages through a shuffled block table, against the flat
           cg_decode_into of the same containers (and checked equal to it).
formats    format 1 (deltas to the group's anchor) against format 2 (deltas
           between adjacent tokens): compression ratio and encode / decode
           GB/s of both on the Llama-2-7B shape (balanced), the Mistral-7B
           shape and the two sweep distributions at C = 1,536 (three levels).

Every figure is fp16 bytes / device time (CUDA events on the launching
stream, inputs resident unless stated, median of `--reps` after `--warmup`).
Status words are checked after every run.  clamp_rate is the share of delta
values whose code hit the [-127, 127] clamp (stats.clamp_counts).
"""
from __future__ import annotations

import argparse
import json
import statistics

import torch

from . import Shape, library
from . import synth
from . import torch_api as ta
from .stats import clamp_counts


def _time(fn, stream, warmup: int, reps: int) -> float:
    for _ in range(warmup):
        fn()
    ts = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    return statistics.median(ts)


def _cell(kv, shape, T, C, level, stream, warmup, reps):
    nch = -(-T // C)
    enc = ta.Encoder(shape, C, nch, kv.device)
    out = torch.empty_like(kv)
    status = ta.new_status(kv.device)
    ms_e = _time(lambda: enc.encode(kv, level, stream=stream), stream, warmup, reps)
    ms_d = _time(lambda: ta.decode_into(enc.out, enc.stride, shape, C, level, nch, out, status,
                                        stream=stream), stream, warmup, reps)
    if ta.status_of(enc.status) != 0 or ta.status_of(status) != 0:
        raise RuntimeError(f"status {ta.status_of(enc.status)} / {ta.status_of(status)}")
    fp16 = kv.numel() * 2
    comp = int(enc.sizes.sum())
    clamped, deltas = clamp_counts(kv, out, C, level)
    return {"C": C, "level": level, "chunks": nch, "encode_ms": round(ms_e, 4),
            "decode_ms": round(ms_d, 4), "encode_gbps": round(fp16 / ms_e / 1e6, 1),
            "decode_gbps": round(fp16 / ms_d / 1e6, 1), "ratio": round(fp16 / comp, 4),
            "clamp_rate": clamped / deltas}


def _gen(w, dev):
    kv = torch.empty((w.L, 2, w.T, w.H, w.D), dtype=torch.int16, device=dev)
    synth.generate_gpu(kv, w.L, w.H, w.D, w.T, w.seed, w.rho, w.p_out, w.m_out)
    torch.cuda.synchronize()
    return kv


def run_grid(names, levels, chunk_sizes, dev, warmup, reps):
    stream = torch.cuda.current_stream(dev)
    for name in names:
        w = synth.WORKLOADS[name]
        kv = _gen(w, dev)
        shape = Shape(w.L, w.H, w.D)
        for C in (chunk_sizes or [w.C]):
            for level in levels:
                res = {"workload": name, **_cell(kv, shape, w.T, C, level, stream, warmup, reps)}
                print(json.dumps(res), flush=True)
        del kv
        torch.cuda.empty_cache()


def run_paged(dev, warmup, reps, page_tokens=16):
    w = synth.WORKLOADS["llama2_7b"]
    kv = _gen(w, dev)
    shape = Shape(w.L, w.H, w.D)
    stream = torch.cuda.current_stream(dev)
    nch, level = w.num_chunks, 1
    enc = ta.encode(kv, w.C, level)
    flat = torch.empty_like(kv)
    status = ta.new_status(dev)
    npages = -(-w.T // page_tokens)
    table = torch.randperm(npages, generator=torch.Generator().manual_seed(0))
    table = table.to(torch.int32).to(dev)
    pool = torch.empty((w.L, 2, npages, page_tokens, w.H, w.D), dtype=torch.int16, device=dev)
    ms_flat = _time(lambda: ta.decode_into(enc.data, enc.stride, shape, w.C, level, nch, flat,
                                           status, stream=stream), stream, warmup, reps)
    ms_paged = _time(lambda: ta.decode_into_paged(enc.data, enc.stride, shape, w.C, level, nch,
                                                  pool, page_tokens, table, w.T, status,
                                                  stream=stream), stream, warmup, reps)
    if ta.status_of(enc.status) != 0 or ta.status_of(status) != 0:
        raise RuntimeError("status")
    # logical token t of the pool: row t % P of page table[t // P]
    logical = pool[:, :, table.long()].reshape(w.L, 2, npages * page_tokens, w.H, w.D)
    same = bool(torch.equal(logical[:, :, :w.T], flat))
    fp16 = kv.numel() * 2
    print(json.dumps({"workload": "llama2_7b_paged", "page_tokens": page_tokens,
                      "pages": npages, "flat_decode_ms": round(ms_flat, 3),
                      "paged_decode_ms": round(ms_paged, 3),
                      "flat_decode_gbps": round(fp16 / ms_flat / 1e6, 1),
                      "paged_decode_gbps": round(fp16 / ms_paged / 1e6, 1),
                      "paged_equals_flat": same}), flush=True)
    if not same:
        raise RuntimeError("paged decode differs from the flat decode")
    del kv, enc, flat, pool, logical
    torch.cuda.empty_cache()


def run_formats(dev, warmup, reps):
    cells = [("llama2_7b", [1]), ("mistral7b", [0, 1, 2]), ("sweep_smooth", [0, 1, 2]),
             ("sweep_rough", [0, 1, 2])]
    stream = torch.cuda.current_stream(dev)
    for name, levels in cells:
        w = synth.WORKLOADS[name]
        kv = _gen(w, dev)
        shape = Shape(w.L, w.H, w.D)
        C = 1536
        nch = -(-w.T // C)
        enc = ta.Encoder(shape, C, nch, dev)
        out = torch.empty_like(kv)
        status = ta.new_status(dev)
        fp16 = kv.numel() * 2
        for level in levels:
            res = {"workload": name, "C": C, "level": level}
            for fmt, adj in (("format1", False), ("format2", True)):
                ms_e = _time(lambda: enc.encode(kv, level, stream=stream, adjacent=adj), stream,
                             warmup, reps)
                ms_d = _time(lambda: ta.decode_into(enc.out, enc.stride, shape, C, level, nch,
                                                    out, status, stream=stream, adjacent=adj),
                             stream, warmup, reps)
                if ta.status_of(enc.status) != 0 or ta.status_of(status) != 0:
                    raise RuntimeError(f"{name} {fmt}: status")
                comp = int(enc.sizes.sum())
                res[fmt] = {"ratio": round(fp16 / comp, 4), "encode_ms": round(ms_e, 3),
                            "decode_ms": round(ms_d, 3),
                            "encode_gbps": round(fp16 / ms_e / 1e6, 1),
                            "decode_gbps": round(fp16 / ms_d / 1e6, 1)}
            print(json.dumps(res), flush=True)
        del kv, enc, out
        torch.cuda.empty_cache()


def run_preencode(dev, warmup, reps, batch=13):
    """Three versions of a batch of chunks ([Practice] 2.1): three single-level
    cg_encode calls against one cg_encode_levels call (one fp16 read)."""
    w = synth.WORKLOADS["llama34b"]
    kv = _gen(w, dev)
    shape = Shape(w.L, w.H, w.D)
    stream = torch.cuda.current_stream(dev)
    single = ta.Encoder(shape, w.C, batch, dev)
    ms_1 = _time(lambda: [single.encode(kv, lv, stream=stream) for lv in range(3)], stream,
                 warmup, reps)
    if ta.status_of(single.status) != 0:
        raise RuntimeError("encode status")
    del single
    torch.cuda.empty_cache()
    lev = ta.LevelsEncoder(shape, w.C, batch, dev)
    ms_3 = _time(lambda: lev.encode(kv, stream=stream), stream, warmup, reps)
    if ta.status_of(lev.status) != 0:
        raise RuntimeError("encode_levels status")
    fp16 = w.L * 2 * batch * w.C * w.H * w.D * 2
    comp = [int(lev.sizes[j * batch:(j + 1) * batch].sum()) for j in range(3)]
    print(json.dumps({"workload": "llama34b_preencode", "chunks": batch, "fp16_bytes": fp16,
                      "ratio_per_level": [round(fp16 / c, 4) for c in comp],
                      "three_encode_ms": round(ms_1, 3), "encode_levels_ms": round(ms_3, 3),
                      "three_encode_gbps": round(fp16 / ms_1 / 1e6, 1),
                      "encode_levels_gbps": round(fp16 / ms_3 / 1e6, 1),
                      "speedup": round(ms_1 / ms_3, 3)}), flush=True)
    del lev, kv
    torch.cuda.empty_cache()


def run_streamed(dev, warmup, reps):
    w = synth.WORKLOADS["llama34b"]
    kv = _gen(w, dev)
    shape = Shape(w.L, w.H, w.D)
    nch = w.num_chunks
    sched = synth.level_schedule(nch, w.seed)
    # pre-encode every chunk at the three levels (device copies for the
    # kernel-only pass, pinned host copies for the streamed pass)
    dev_c, host_c = {}, {}
    for level in range(3):
        enc = ta.encode(kv, w.C, level)
        torch.cuda.synchronize()
        if ta.status_of(enc.status) != 0:
            raise RuntimeError("encode status")
        sizes = enc.sizes.cpu().tolist()
        for k in range(nch):
            if sched[k] != level:
                continue
            n = ((sizes[k] + 15) // 16) * 16
            dev_c[k] = enc.data[k * enc.stride:k * enc.stride + n].clone()
            hb = torch.empty(n, dtype=torch.uint8, pin_memory=True)
            hb.copy_(dev_c[k])
            host_c[k] = hb
        del enc
    comp_bytes = sum(host_c[k].numel() for k in range(nch))
    fp16 = kv.numel() * 2
    out = torch.empty_like(kv)
    status = ta.new_status(dev)
    comp = torch.cuda.Stream(dev)

    def kernel_only():
        for k in range(nch):
            ta.decode_into(dev_c[k], dev_c[k].numel(), shape, w.C, sched[k], 1, out, status,
                           stream=comp)

    maxb = max(b.numel() for b in host_c.values())
    stage = [torch.empty(maxb, dtype=torch.uint8, device=dev) for _ in range(2)]
    copy = torch.cuda.Stream(dev)
    ready = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]

    def streamed():
        for k in range(nch):
            s = k % 2
            buf = host_c[k]
            with torch.cuda.stream(copy):
                copy.wait_event(done[s])
                stage[s][:buf.numel()].copy_(buf, non_blocking=True)
                ready[s].record(copy)
            comp.wait_event(ready[s])
            ta.decode_into(stage[s], stage[s].numel(), shape, w.C, sched[k], 1, out, status,
                           stream=comp)
            done[s].record(comp)

    def timed(fn):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(comp)
            fn()
            # the streamed pass ends when its last decode ends (on `comp`)
            e1.record(comp)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return statistics.median(ts)

    ms_k = timed(kernel_only)
    ms_s = timed(streamed)
    if ta.status_of(status) != 0:
        raise RuntimeError("decode status")
    levels = {lv: sum(1 for x in sched if x == lv) for lv in range(3)}
    print(json.dumps({"workload": "llama34b", "chunks": nch, "chunks_per_level": levels,
                      "container_bytes": comp_bytes, "fp16_bytes": fp16,
                      "ratio": round(fp16 / comp_bytes, 4),
                      "decode_kernel_only_ms": round(ms_k, 3),
                      "decode_kernel_only_gbps": round(fp16 / ms_k / 1e6, 1),
                      "decode_streamed_ms": round(ms_s, 3),
                      "decode_streamed_gbps": round(fp16 / ms_s / 1e6, 1),
                      "h2d_gbps_during_stream": round(comp_bytes / ms_s / 1e6, 1)}), flush=True)


def main() -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--config", choices=["mistral7b", "sweep", "llama34b", "formats", "paged"],
                    required=True)
    ap.add_argument("--warmup", type=int, default=2)
    ap.add_argument("--reps", type=int, default=5)
    args = ap.parse_args()
    library()
    dev = torch.device("cuda", 0)
    if args.config == "mistral7b":
        run_grid(["mistral7b"], [0, 1, 2], None, dev, args.warmup, args.reps)
    elif args.config == "sweep":
        w = synth.WORKLOADS["sweep_smooth"]
        run_grid(["sweep_smooth", "sweep_rough"], [0, 1, 2], list(w.chunk_sizes), dev,
                 args.warmup, args.reps)
    elif args.config == "formats":
        run_formats(dev, args.warmup, args.reps)
    elif args.config == "paged":
        run_paged(dev, args.warmup, args.reps)
    else:
        run_preencode(dev, args.warmup, args.reps)
        run_streamed(dev, args.warmup, args.reps)
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
