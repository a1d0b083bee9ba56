"""Command-line round trip of the codec on one of the synthetic workloads.

    python -m kv_cache_compression_cachegen_b200.roundtrip --workload mistral7b --level 1

Generates the workload's KV cache on the GPU, then runs cg_encode of all its
chunks followed by cg_decode_into of all containers, `--repeat` times, and
prints the per-phase device times, the compression ratio and the status
words.  Useful as a quick check of a build and as a small, fixed command for
profilers.  `--format 2` uses the adjacent-token format (cg_encode_adjacent,
cg_decode_adjacent_into); `--levels` encodes with cg_encode_levels (all three
levels from one pass) and decodes the `--level` set.
"""
from __future__ import annotations

import argparse
import json

import torch

from . import (Shape, cg_decode_adjacent_into, cg_decode_into, cg_encode, cg_encode_adjacent,
               cg_encode_levels, check, library)
from . import synth
from . import torch_api as ta


def main() -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="mistral7b", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--level", type=int, default=1)
    ap.add_argument("--chunk", type=int, default=0, help="chunk size (default: the workload's)")
    ap.add_argument("--tokens", type=int, default=0, help="sequence length (default: workload's)")
    ap.add_argument("--repeat", type=int, default=2)
    ap.add_argument("--format", type=int, default=1, choices=[1, 2])
    ap.add_argument("--levels", action="store_true")
    args = ap.parse_args()
    if args.levels and args.format != 1:
        ap.error("--levels encodes format 1")
    library()
    w = synth.WORKLOADS[args.workload]
    T = args.tokens or w.T
    C = args.chunk or w.C
    L, H, D = w.L, w.H, w.D
    nch = -(-T // C)
    dev = torch.device("cuda", 0)
    kv = torch.empty((L, 2, T, H, D), dtype=torch.int16, device=dev)
    synth.generate_gpu(kv, L, H, D, T, w.seed, w.rho, w.p_out, w.m_out)
    shape = Shape(L, H, D)
    enc = ta.LevelsEncoder(shape, C, nch, dev) if args.levels else ta.Encoder(shape, C, nch, dev)
    out = torch.empty_like(kv)
    status = ta.new_status(dev)
    stream = torch.cuda.current_stream(dev)
    # the containers the decode reads (the --level set of a three-level encode)
    lv_off = args.level * nch * enc.stride if args.levels else 0
    dec_in = enc.out[lv_off:lv_off + nch * enc.stride]
    sizes = enc.sizes[args.level * nch:(args.level + 1) * nch] if args.levels else enc.sizes
    times = []
    for _ in range(args.repeat):
        e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        e0.record(stream)
        if args.levels:
            check(cg_encode_levels(shape, kv, T, 0, nch, C, enc.out, enc.stride, enc.sizes,
                                   enc.status, enc.workspace, enc.ws_bytes, stream),
                  "cg_encode_levels")
        elif args.format == 2:
            check(cg_encode_adjacent(shape, kv, T, 0, nch, C, args.level, enc.out, enc.stride,
                                     enc.sizes, enc.status, enc.workspace, enc.ws_bytes, stream),
                  "cg_encode_adjacent")
        else:
            check(cg_encode(shape, kv, T, 0, nch, C, args.level, None, enc.out, enc.stride,
                            enc.sizes, enc.status, enc.workspace, enc.ws_bytes, stream),
                  "cg_encode")
        e1.record(stream)
        dec = cg_decode_adjacent_into if args.format == 2 else cg_decode_into
        check(dec(shape, dec_in, enc.stride, nch, C, args.level, out, T, status, stream),
              dec.__name__)
        e2.record(stream)
        torch.cuda.synchronize(dev)
        times.append((e0.elapsed_time(e1), e1.elapsed_time(e2)))
    comp = int(sizes.sum().item())
    res = {"workload": args.workload, "L": L, "H": H, "D": D, "T": T, "C": C, "chunks": nch,
           "level": args.level, "format": args.format, "levels_encode": args.levels,
           "fp16_bytes": kv.numel() * 2, "container_bytes": comp,
           "ratio": round(kv.numel() * 2 / comp, 4),
           "encode_ms": [round(a, 4) for a, _ in times],
           "decode_ms": [round(b, 4) for _, b in times],
           "encode_status": ta.status_of(enc.status), "decode_status": ta.status_of(status)}
    print(json.dumps(res))
    return 0 if res["encode_status"] == 0 and res["decode_status"] == 0 else 1


if __name__ == "__main__":
    raise SystemExit(main())
