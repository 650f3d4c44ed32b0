"""The C-ABI library builds, loads and exports every symbol include/star.h
declares; argument validation rejects bad calls before anything launches.
These run without a GPU."""
import ctypes
import os
import re

import pytest
import torch

from block_sparse_long_rope_b200 import _abi
from block_sparse_long_rope_b200 import build as star_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "star.h")

OK, INVALID, UNSUPPORTED, CUDA = 0, 1, 2, 3
FAKE = ctypes.c_void_p(0x10000)   # aligned, never dereferenced: validation fails first
ODD = ctypes.c_void_p(0x10008)    # not 16-byte aligned
NULL = ctypes.c_void_p(0)


@pytest.fixture(scope="module")
def lib():
    star_build.build()
    return _abi.load()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(star_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_four_hot_path_calls():
    names = _declared_functions()
    for n in ("star_rope", "star_phase1_encode", "star_phase2_partial", "star_lse_merge"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert set(names) == set(_abi.EXPORTS)
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_empty_error(lib):
    assert b"sm_100a" in lib.star_version()


def test_loaded_library_was_built_from_these_sources(lib):
    # the build digest (sources, headers, flags) ends the version string
    assert star_build.loaded_matches_sources(), lib.star_version()


def test_phase2_workspace_size_formula(lib):
    # star_phase2_workspace_bytes(B, T, Hq, Hkv, D, Lcap, block_len): the decode
    # path's partials depend on Hkv (one 16-row tile per GQA group) and on the
    # cache capacity (the splits a context of up to Lcap rows can have)
    up = lambda x: -(-x // 256) * 256  # noqa: E731
    for B, Hq, Hkv, D, Lcap, b in [(1, 32, 8, 128, 16384 + 192, 4096), (2, 4, 1, 64, 2072, 512),
                                   (1, 64, 8, 128, 131072 + 384, 32768)]:
        nsplit_cap = -(-Lcap // b) + 1
        header = 256 + up(B * Hkv * nsplit_cap * 4) + up(B * Hkv * 4)
        splits = B * Hkv * nsplit_cap
        units = max(512, splits) + splits
        rows = units * 16
        dec = header + up(B * 1 * Hq * D * 2) + up(rows * D * 4) + up(rows * 4)
        assert lib.star_phase2_workspace_bytes(B, 1, Hq, Hkv, D, Lcap, b) == dec


def _subsplits(B, Hq, Hkv, T, L, b):
    """Sub-splits per block of a query chunk: fill one wave of 148 CTAs with
    (split, query tile, head group) items, equal 128-key multiples, at most 4."""
    if L % b:
        return 1
    n = L // b
    g = Hq // Hkv
    hpc = 2 if g % 2 == 0 else 1
    per_split = B * Hkv * (g // hpc) * -(-T // 128)
    if (n + 1) * per_split >= 148:
        return 1
    nsub = min(4, (148 - per_split) // (n * per_split))
    while nsub > 1 and b % (nsub * 128):
        nsub -= 1
    return max(1, nsub)


def _chunk_scratch(B, T, Hq, Hkv, D, Lcap, b):
    up = lambda x: -(-x // 256) * 256  # noqa: E731
    best = 0
    for n in range(1, Lcap // b + 1):
        ns = _subsplits(B, Hq, Hkv, T, n * b, b)
        if ns > 1:
            rows = B * Hq * (n * ns) * T  # the context sub-splits (the tail is written in place)
            best = max(best, up(rows * D * 4) + up(rows * 4))
    return best


def test_query_chunk_subsplit_rule():
    # llama8b-16k query chunk: 80 items -> 2 sub-splits per block, 144 items
    assert _subsplits(1, 32, 8, 128, 16384, 4096) == 2
    # enough items already (llama70b-128k, 256 tokens): no cut
    assert _subsplits(1, 64, 8, 256, 131072, 32768) == 1
    # a ragged context is never cut
    assert _subsplits(1, 32, 8, 128, 16000, 4096) == 1


def test_workspace_sizes(lib):
    # Phase 1: status header + rotated Q (bf16)
    assert lib.star_phase1_workspace_bytes(1, 2048, 4, 64) == 256 + 2048 * 4 * 64 * 2
    assert lib.star_phase1_workspace_bytes(2, 1000, 3, 128) >= 256 + 2 * 1000 * 3 * 128 * 2
    # Phase 2 query chunk (tensor-core path): the decode header (status block,
    # split and head counters, kept on every Phase-2 path) + rotated q only
    chunk = lib.star_phase2_workspace_bytes(1, 128, 32, 8, 128, 16384 + 192, 4096)
    splits = -(-(16384 + 192) // 4096) + 1
    header = 256 + (-(-(8 * splits * 4) // 256)) * 256 + 256
    assert chunk == header + 128 * 32 * 128 * 2 + _chunk_scratch(1, 128, 32, 8, 128, 16384 + 192, 4096)
    # decode path adds chunk scratch
    dec = lib.star_phase2_workspace_bytes(1, 1, 32, 8, 128, 16384 + 192, 4096)
    assert dec > 256 + 32 * 128 * 2
    assert lib.star_phase2_workspace_bytes(0, 1, 1, 1, 64, 10, 10) == 256


def _p1(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, kc=FAKE, vc=FAKE, Lcap=64, lse=NULL, B=1, L=64,
             Hq=4, Hkv=2, D=64, b=16, a=16, theta=1e4, ws=FAKE, wsb=1 << 30)
    a.update(kw)
    return lib.star_phase1_encode(a["q"], a["k"], a["v"], a["o"], a["kc"], a["vc"], a["Lcap"],
                                  a["lse"], a["B"], a["L"], a["Hq"], a["Hkv"], a["D"], a["b"],
                                  a["a"], a["theta"], a["ws"], a["wsb"], NULL)


@pytest.mark.parametrize("kw,status", [
    (dict(q=NULL), INVALID),
    (dict(o=ODD), INVALID),
    (dict(Hq=5, Hkv=2), INVALID),          # Hq % Hkv != 0
    (dict(D=96), UNSUPPORTED),
    (dict(a=17), INVALID),                 # anchor_len > block_len
    (dict(a=-1), INVALID),
    (dict(b=0), INVALID),
    (dict(L=0), INVALID),
    (dict(Lcap=63), INVALID),              # Lcap < L
    (dict(wsb=100), INVALID),              # workspace too small
    (dict(theta=0.0), INVALID),
    (dict(lse=ctypes.c_void_p(0x10002)), INVALID),
])
def test_phase1_validation(lib, kw, status):
    assert _p1(lib, **kw) == status
    assert lib.star_last_error()  # a message is kept


def test_ext_workspace_sizes(lib):
    base = lib.star_phase1_workspace_bytes(1, 2048, 4, 64)
    assert lib.star_phase1_ext_workspace_bytes(1, 2048, 4, 2, 64, 0) == base
    # + the gathered table's K and V, bf16 [B, Hkv, G, D] each
    assert lib.star_phase1_ext_workspace_bytes(1, 2048, 4, 2, 64, 100) == base + 2 * 100 * 2 * 64 * 2
    assert lib.star_phase1_ext_workspace_bytes(1, 2048, 4, 2, 64, -1) == 256


def _p1x(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, kc=FAKE, vc=FAKE, Lcap=64, lse=NULL, B=1, L=64,
             Hq=4, Hkv=2, D=64, b=16, src=FAKE, pos=FAKE, G=8, bounds=FAKE, xk=NULL, xv=NULL,
             NX=0, pos0=0, theta=1e4, ws=FAKE, wsb=1 << 30)
    a.update(kw)
    return lib.star_phase1_encode_ext(a["q"], a["k"], a["v"], a["o"], a["kc"], a["vc"], a["Lcap"],
                                      a["lse"], a["B"], a["L"], a["Hq"], a["Hkv"], a["D"], a["b"],
                                      a["src"], a["pos"], a["G"], a["bounds"], a["xk"], a["xv"],
                                      a["NX"], a["pos0"], a["theta"], a["ws"], a["wsb"], NULL)


@pytest.mark.parametrize("kw,status", [
    (dict(G=-1), INVALID),
    (dict(src=NULL), INVALID),             # G > 0 needs the table
    (dict(pos=NULL), INVALID),
    (dict(bounds=NULL), INVALID),
    (dict(src=ctypes.c_void_p(0x10002)), INVALID),
    (dict(NX=-1), INVALID),
    (dict(NX=2), INVALID),                 # extra rows without buffers
    (dict(NX=2, xk=FAKE, xv=ODD), INVALID),
    (dict(wsb=256 + 64 * 4 * 64 * 2), INVALID),  # room for Q only, not the table
    (dict(D=96), UNSUPPORTED),
    (dict(Lcap=63), INVALID),
    (dict(pos0=-1), INVALID),
    (dict(pos0=2**31 - 10), INVALID),      # ctx_pos0 + L past int32
])
def test_phase1_ext_validation(lib, kw, status):
    assert _p1x(lib, **kw) == status
    assert lib.star_last_error()


def _p2(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, T=1, kc=FAKE, vc=FAKE, Lcap=100, L=64, b=16, tail=0,
             po=FAKE, pl=FAKE, B=1, Hq=4, Hkv=2, D=64, theta=1e4, ws=FAKE, wsb=1 << 30)
    a.update(kw)
    ns = ctypes.c_int(-1)
    return lib.star_phase2_partial(a["q"], a["k"], a["v"], a["T"], a["kc"], a["vc"], a["Lcap"],
                                   a["L"], a["b"], a["tail"], a["po"], a["pl"], ctypes.byref(ns),
                                   a["B"], a["Hq"], a["Hkv"], a["D"], a["theta"], a["ws"],
                                   a["wsb"], NULL)


@pytest.mark.parametrize("kw,status", [
    (dict(T=0), INVALID),
    (dict(tail=-1), INVALID),
    (dict(Lcap=64, T=1), INVALID),         # no room for the new token
    (dict(L=60, tail=30, T=11), INVALID),  # L + tail + T > Lcap
    (dict(pl=NULL), INVALID),
    (dict(po=ODD), INVALID),
    (dict(D=80), UNSUPPORTED),
    (dict(Hkv=3), INVALID),
    (dict(wsb=16), INVALID),
])
def test_phase2_validation(lib, kw, status):
    assert _p2(lib, **kw) == status


def _p2x(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, T=1, kc=FAKE, vc=FAKE, Lcap=100, L=64, b=16, tail=0,
             pos0=1000, qpos0=1064, with_tail=1, po=FAKE, pl=FAKE, B=1, Hq=4, Hkv=2, D=64,
             theta=1e4, ws=FAKE, wsb=1 << 30)
    a.update(kw)
    ns = ctypes.c_int(-1)
    return lib.star_phase2_partial_ext(a["q"], a["k"], a["v"], a["T"], a["kc"], a["vc"], a["Lcap"],
                                       a["L"], a["b"], a["tail"], a["pos0"], a["qpos0"],
                                       a["with_tail"], a["po"], a["pl"], ctypes.byref(ns), a["B"],
                                       a["Hq"], a["Hkv"], a["D"], a["theta"], a["ws"], a["wsb"],
                                       NULL)


@pytest.mark.parametrize("kw,status", [
    (dict(qpos0=1065), INVALID),                     # the tail must follow the cache
    (dict(with_tail=2), INVALID),
    (dict(with_tail=0, tail=3), INVALID),            # no tail split, no tail tokens
    (dict(pos0=-1, qpos0=63), INVALID),
    (dict(with_tail=0, qpos0=2**31 - 1), INVALID),   # q_pos0 + T past int32
    (dict(k=NULL), INVALID),                         # the tail needs the new k/v
    (dict(Lcap=64), INVALID),                        # no room for the new token
    (dict(D=80), UNSUPPORTED),
])
def test_phase2_ext_validation(lib, kw, status):
    assert _p2x(lib, **kw) == status
    assert lib.star_last_error()


def test_merge_ranks_validation(lib):
    ns2 = (ctypes.c_int * 2)(3, 4)
    ok_args = (FAKE, FAKE, 2, ns2, 4, FAKE, NULL, 1, 1, 4, 64, NULL)
    assert lib.star_lse_merge_ranks(*((FAKE, FAKE, 0) + ok_args[3:])) == INVALID      # no ranks
    assert lib.star_lse_merge_ranks(*((FAKE, FAKE, 65) + ok_args[3:])) == INVALID     # > 64 ranks
    assert lib.star_lse_merge_ranks(*(ok_args[:4] + (3,) + ok_args[5:])) == INVALID   # 4 > stride 3
    assert lib.star_lse_merge_ranks(*(ok_args[:3] + (None,) + ok_args[4:])) == INVALID
    zero = (ctypes.c_int * 2)(0, 0)
    assert lib.star_lse_merge_ranks(*(ok_args[:3] + (zero,) + ok_args[4:])) == INVALID  # nothing
    assert lib.star_lse_merge_ranks(*(ok_args[:10] + (32, NULL))) == UNSUPPORTED


def test_stack_calls_validation(lib):
    # RMSNorm: dm a multiple of 8, aligned non-NULL pointers, eps >= 0
    assert lib.star_rmsnorm(FAKE, FAKE, FAKE, 4, 12, 1e-5, NULL) == INVALID
    assert lib.star_rmsnorm(FAKE, FAKE, FAKE, -1, 64, 1e-5, NULL) == INVALID
    assert lib.star_rmsnorm(FAKE, NULL, FAKE, 4, 64, 1e-5, NULL) == INVALID
    assert lib.star_rmsnorm(FAKE, FAKE, ODD, 4, 64, 1e-5, NULL) == INVALID
    assert lib.star_rmsnorm(FAKE, FAKE, FAKE, 4, 64, -1.0, NULL) == INVALID
    # linear: N, K multiples of 8, accumulate 0/1, aligned workspace
    assert lib.star_linear(FAKE, FAKE, FAKE, 4, 12, 64, 0, NULL, 0, NULL) == INVALID
    assert lib.star_linear(FAKE, FAKE, FAKE, 4, 64, 60, 0, NULL, 0, NULL) == INVALID
    assert lib.star_linear(FAKE, FAKE, FAKE, 0, 64, 64, 0, NULL, 0, NULL) == INVALID
    assert lib.star_linear(FAKE, FAKE, FAKE, 4, 64, 64, 2, NULL, 0, NULL) == INVALID
    assert lib.star_linear(NULL, FAKE, FAKE, 4, 64, 64, 0, NULL, 0, NULL) == INVALID
    assert lib.star_linear(FAKE, FAKE, FAKE, 4, 64, 64, 0, NULL, 1024, NULL) == INVALID
    assert lib.star_linear(FAKE, FAKE, FAKE, 4, 64, 64, 0, ODD, 1024, NULL) == INVALID
    assert lib.star_linear(FAKE, FAKE, FAKE, 4, 64, 64, 0, NULL, 0, NULL) == INVALID  # no status word
    assert lib.star_linear(FAKE, FAKE, FAKE, 4, 64, 64, 0, FAKE, 128, NULL) == INVALID
    assert lib.star_last_error()
    # linear_rope: head_dim 64/128, whole heads, M = B * seq_len, cache rows >= seq_len
    def lr(M=8, N=128, K=64, hd=64, rot=1, S=4, pos0=0, theta=1e4, rows=0, ws=FAKE, wsb=256):
        return lib.star_linear_rope(FAKE, FAKE, FAKE, M, N, K, hd, rot, S, pos0, theta, rows, ws,
                                    wsb, NULL)
    assert lr(hd=96) == UNSUPPORTED
    assert lr(N=96) == INVALID            # 1.5 heads of 64
    assert lr(S=3) == INVALID             # M not a multiple of seq_len
    assert lr(rows=3) == INVALID          # cache shorter than a sequence
    assert lr(rot=0, rows=0) == INVALID   # nothing to do beyond star_linear
    assert lr(rot=2) == INVALID
    assert lr(pos0=-1) == INVALID
    assert lr(theta=0.0) == INVALID
    assert lr(ws=NULL, wsb=0) == INVALID
    assert lr(wsb=256) == INVALID         # rotation needs room for the cos/sin table
    assert lib.star_last_error()
    # status word, then the fp32 (cos, sin) of seq_len positions x head_dim/2 frequencies
    assert lib.star_linear_rope_workspace_bytes(4096, 128, 1) == 256 + 4096 * 64 * 8
    assert lib.star_linear_rope_workspace_bytes(5, 64, 1) == 256 + 5 * 32 * 8
    assert lib.star_linear_rope_workspace_bytes(4096, 128, 0) == 256
    # K/V projection into the caches: whole heads, cache rows >= seq_len, both caches given
    def kv(N=128, hd=64, S=4, rows=8, vc=FAKE, ws=FAKE, wsb=1 << 20):
        return lib.star_linear_kv_cache(FAKE, FAKE, FAKE, vc, 8, N, 64, hd, S, 0, 1e4, rows, ws,
                                        wsb, NULL)
    assert kv(hd=96) == UNSUPPORTED
    assert kv(N=96) == INVALID
    assert kv(rows=3) == INVALID
    assert kv(vc=NULL) == INVALID
    assert kv(vc=ODD) == INVALID
    assert kv(wsb=256) == INVALID         # no room for the cos/sin table


def test_phase1_rotated_validation(lib):
    def p1r(q=FAKE, o=FAKE, kc=FAKE, vc=FAKE, Lcap=64, lse=NULL, B=1, L=64, Hq=4, Hkv=2, D=64,
            b=16, a=16, ws=FAKE, wsb=256):
        return lib.star_phase1_encode_rotated(q, o, kc, vc, Lcap, lse, B, L, Hq, Hkv, D, b, a,
                                              ws, wsb, NULL)
    assert p1r(q=NULL) == INVALID
    assert p1r(kc=ODD) == INVALID
    assert p1r(a=17) == INVALID
    assert p1r(Lcap=63) == INVALID
    assert p1r(wsb=255) == INVALID        # the status word needs 256 bytes
    assert p1r(D=80) == UNSUPPORTED
    assert p1r(Hq=3) == INVALID


def test_merge_and_rope_validation(lib):
    assert lib.star_lse_merge(FAKE, FAKE, 0, FAKE, NULL, 1, 1, 1, 64, NULL) == INVALID
    assert lib.star_lse_merge(FAKE, FAKE, 2, FAKE, NULL, 1, 1, 1, 32, NULL) == UNSUPPORTED
    assert lib.star_lse_merge(NULL, FAKE, 2, FAKE, NULL, 1, 1, 1, 64, NULL) == INVALID
    s8 = (ctypes.c_int64 * 3)(8, 8, 8)
    s5 = (ctypes.c_int64 * 3)(8, 5, 8)
    assert lib.star_rope(FAKE, s5, FAKE, s8, NULL, 0, 1, 1, 1, 64, 1e4, NULL) == INVALID
    assert lib.star_rope(FAKE, s8, FAKE, s8, NULL, 0, 1, 1, 1, 48, 1e4, NULL) == UNSUPPORTED
    assert lib.star_rope(ODD, s8, FAKE, s8, NULL, 0, 1, 1, 1, 64, 1e4, NULL) == INVALID
    assert lib.star_debug_index(10, 4, 5, FAKE, FAKE, FAKE, NULL) == INVALID


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path only")
def test_valid_call_without_device_reports_cuda_error(lib):
    # every argument is valid; with no CUDA device the device probe fails
    # and the call returns an error instead of launching
    assert _p1(lib) in (CUDA, UNSUPPORTED)
    assert lib.star_last_error()
    assert _p1x(lib, G=0, src=NULL, pos=NULL, bounds=NULL) in (CUDA, UNSUPPORTED)
    assert _p2x(lib) in (CUDA, UNSUPPORTED)
    assert _p2x(lib, with_tail=0, k=NULL, v=NULL, qpos0=5000) in (CUDA, UNSUPPORTED)
    assert lib.star_linear(FAKE, FAKE, FAKE, 4, 64, 64, 0, FAKE, 256, NULL) in (CUDA, UNSUPPORTED)
    assert lib.star_phase1_encode_rotated(FAKE, FAKE, FAKE, FAKE, 64, NULL, 1, 64, 4, 2, 64, 16,
                                          16, FAKE, 256, NULL) in (CUDA, UNSUPPORTED)


def test_python_binding_raises_on_missing_library(tmp_path):
    saved = _abi._lib
    try:
        _abi._lib = None
        with pytest.raises(RuntimeError, match="missing"):
            _abi.load(str(tmp_path / "nope.so"))
    finally:
        _abi._lib = saved


def test_wait_probe_validation(lib):
    assert lib.star_debug_wait_probe(NULL, 0.05, NULL) == INVALID
    assert lib.star_debug_wait_probe(FAKE, 0.0, NULL) == INVALID
    assert lib.star_debug_wait_probe(FAKE, 3.0, NULL) == INVALID
