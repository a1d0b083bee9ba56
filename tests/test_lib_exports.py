"""The native libraries build, load and export every declared entry point; the
pure-host queries agree with the oracle.  No GPU is needed."""
import ctypes
import re
from pathlib import Path

import numpy as np
import pytest

ROOT = Path(__file__).resolve().parents[1]


def _declared(header: Path):
    text = header.read_text(encoding="utf-8")
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(cg_[a-z_]+)\s*\(", text)))


def test_header_declares_the_calls():
    names = _declared(ROOT / "include" / "cachegen.h")
    for need in ("cg_build_tables", "cg_encode", "cg_decode", "cg_decode_into"):
        assert need in names


def test_codec_library_exports_every_declared_symbol(native_built):
    import kv_cache_compression_cachegen_b200 as cg
    lib = ctypes.CDLL(str(cg.library_path()))
    for header in (ROOT / "include").glob("*.h"):
        for name in _declared(header):
            assert hasattr(lib, name), name


def test_synth_library_exports(native_built):
    from kv_cache_compression_cachegen_b200 import synth
    lib = ctypes.CDLL(str(synth._LIB))
    assert hasattr(lib, "kvsynth_generate")


@pytest.mark.parametrize("L,H,D,n", [(1, 1, 16, 10), (32, 8, 128, 1536), (32, 32, 128, 1536),
                                     (48, 8, 128, 7), (4, 2, 64, 256)])
def test_host_size_queries_match_oracle(native_built, oracle_lib, L, H, D, n):
    import kv_cache_compression_cachegen_b200 as cg
    assert cg.cg_section_offsets((L, H, D), n) == oracle_lib.sections(L, H, D, n)
    assert cg.cg_encoded_bound((L, H, D), n) == oracle_lib.encoded_bound(L, H, D, n)
    secs = oracle_lib.sections(L, H, D, 1)
    assert cg.cg_tables_bytes((L, H, D)) == secs[2] + L * 2 * H * 512 - 64


def test_argument_errors_are_synchronous(native_built):
    import kv_cache_compression_cachegen_b200 as cg
    shp = (4, 2, 64)
    assert cg.library().cg_encoded_bound(ctypes.byref(cg.Shape(4, 2, 40)), 256,
                                         ctypes.byref(ctypes.c_uint64())) == cg.CG_ERR_UNSUPPORTED
    assert cg.cg_encode(shp, None, 256, 0, 1, 256, 1, None, None, 0, None, None, None, 0,
                        stream=0) == cg.CG_ERR_INVALID_ARG
    assert cg.cg_decode(shp, None, 64, 1, 256, 1, None, 0, None, stream=0) == cg.CG_ERR_INVALID_ARG
    assert cg.cg_decode_into(shp, 16, 64, 1, 256, 5, 16, 256, 16, stream=0) == cg.CG_ERR_INVALID_ARG
    assert cg.cg_build_tables(shp, 16, 256, 0, 2, 256, 1, 16, 16, stream=0) == cg.CG_ERR_INVALID_ARG
    # empty calls: no chunk, no token
    assert cg.cg_encode(shp, 16, 256, 0, 0, 256, 1, None, 16, 4096, 16, 16, 256, 1 << 20,
                        stream=0) == cg.CG_ERR_INVALID_ARG
    assert cg.cg_encode(shp, 16, 0, 0, 1, 256, 1, None, 16, 4096, 16, 16, 256, 1 << 20,
                        stream=0) == cg.CG_ERR_INVALID_ARG
    assert cg.cg_decode(shp, 16, 4096, 0, 256, 1, 16, 1 << 20, 16, stream=0) == cg.CG_ERR_INVALID_ARG
    assert cg.cg_decode_into(shp, 16, 4096, 1, 256, 1, 16, 0, 16, stream=0) == cg.CG_ERR_INVALID_ARG
    # paged decode: no block table, or an empty pool
    assert cg.cg_decode_into_paged(shp, 16, 64, 1, 256, 1, 16, 4, 16, None, 64, 16,
                                   stream=0) == cg.CG_ERR_INVALID_ARG
    assert cg.cg_decode_into_paged(shp, 16, 64, 1, 256, 1, 16, 0, 16, 16, 64, 16,
                                   stream=0) == cg.CG_ERR_INVALID_ARG
    assert cg.cg_status_string(cg.CG_ERR_CORRUPT) == "corrupt container"


def test_encode_levels_argument_checks(native_built):
    import kv_cache_compression_cachegen_b200 as cg
    shp = (4, 2, 64)
    one = cg.cg_encode_workspace_bytes(shp, 256, 3)
    three = cg.cg_encode_levels_workspace_bytes(shp, 256, 3)
    # three symbol arrays and constant sets, one set of stream slots
    assert one < three < 3 * one
    bound = cg.cg_encoded_bound(shp, 256)
    # missing pointers, no chunk, unaligned workspace: rejected before any launch
    assert cg.cg_encode_levels(shp, None, 256, 0, 1, 256, 16, bound, 16, 16, 256, three,
                               stream=0) == cg.CG_ERR_INVALID_ARG
    assert cg.cg_encode_levels(shp, 16, 256, 0, 0, 256, 16, bound, 16, 16, 256, three,
                               stream=0) == cg.CG_ERR_INVALID_ARG
    assert cg.cg_encode_levels(shp, 16, 256, 0, 1, 256, 16, bound, 16, 16, 16, three,
                               stream=0) == cg.CG_ERR_INVALID_ARG
    # a workspace sized for one level, or an out stride without room for the tables
    assert cg.cg_encode_levels(shp, 16, 256, 0, 1, 256, 16, bound, 16, 16, 256,
                               cg.cg_encode_workspace_bytes(shp, 256, 1),
                               stream=0) == cg.CG_ERR_CAPACITY
    assert cg.cg_encode_levels(shp, 16, 256, 0, 1, 256, 16, 64, 16, 16, 256, three,
                               stream=0) == cg.CG_ERR_CAPACITY


def test_adjacent_format_argument_checks(native_built):
    import kv_cache_compression_cachegen_b200 as cg
    shp = (4, 2, 64)
    ws = cg.cg_encode_workspace_bytes(shp, 256, 1)
    bound = cg.cg_encoded_bound(shp, 256)
    assert cg.cg_encode_adjacent(shp, None, 256, 0, 1, 256, 1, 16, bound, 16, 16, 256, ws,
                                 stream=0) == cg.CG_ERR_INVALID_ARG
    assert cg.cg_encode_adjacent(shp, 16, 256, 0, 1, 256, 3, 16, bound, 16, 16, 256, ws,
                                 stream=0) == cg.CG_ERR_INVALID_ARG
    assert cg.cg_encode_adjacent(shp, 16, 256, 0, 1, 256, 1, 16, bound, 16, 16, 256, ws - 256,
                                 stream=0) == cg.CG_ERR_CAPACITY
    assert cg.cg_decode_adjacent(shp, None, 64, 1, 256, 1, 16, 1 << 20, 16,
                                 stream=0) == cg.CG_ERR_INVALID_ARG
    assert cg.cg_decode_adjacent(shp, 16, 4096, 1, 256, 1, 16, 16, 16,
                                 stream=0) == cg.CG_ERR_CAPACITY
    assert cg.cg_decode_adjacent_into(shp, 16, 4096, 1, 256, 1, 16, 0, 16,
                                      stream=0) == cg.CG_ERR_INVALID_ARG
    # the two-pass grid of a huge call is refused up front
    assert cg.cg_decode_adjacent((1024, 64, 256), 16, 4096, 100, 16384, 1, 16, 1 << 62, 16,
                                 stream=0) in (cg.CG_ERR_UNSUPPORTED, cg.CG_ERR_CAPACITY)


def test_binding_signatures_match_the_header():
    # every ctypes signature of the binding has as many arguments as the
    # prototype declared in include/cachegen.h
    import kv_cache_compression_cachegen_b200 as cg
    text = re.sub(r"/\*.*?\*/", "", (ROOT / "include" / "cachegen.h").read_text(encoding="utf-8"),
                  flags=re.S)
    protos = {}
    for m in re.finditer(r"\b(cg_[a-z_]+)\s*\(([^;{]*?)\)\s*;", text, flags=re.S):
        args = [a for a in m.group(2).split(",") if a.strip() and a.strip() != "void"]
        protos[m.group(1)] = len(args)
    assert set(cg._SIGNATURES) == set(protos), set(cg._SIGNATURES) ^ set(protos)
    for name, (_, argtypes) in cg._SIGNATURES.items():
        assert len(argtypes) == protos[name], (name, len(argtypes), protos[name])
