"""Host-side planning of the decode kernel (star_plan.h, built here for the
host): the keys per work unit and the units per split for many shapes and SM
counts. The decode scratch in every Phase-2 workspace is sized for
decode_units_bound units, and the kernel's split counters for at most
kMaxChunksPerSplit units per split; a plan outside either bound would write
past the workspace, so both are checked over a sweep that includes ragged
last blocks, long tails, many splits and small and large GPUs."""
import ctypes
import itertools
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_sparse_long_rope_b200", "csrc")
INCLUDE = os.path.join(ROOT, "include")


@pytest.fixture(scope="module")
def lib(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("dp") / "libdp.so")
    subprocess.check_call(["/usr/local/cuda/bin/nvcc", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
                           "-I" + CSRC, "-I" + INCLUDE,
                           os.path.join(ROOT, "tests", "harness", "decode_plan.cu"), "-o", out])
    lb = ctypes.CDLL(out)
    lb.dp_units_bound.restype = ctypes.c_longlong
    return lb


SHAPES = list(itertools.product(
    [1, 2, 4],                              # B
    [1, 2, 8],                              # Hkv
    [(16384, 4096), (16000, 4096), (65536, 16384), (131072, 32768), (1048576, 131072),
     (2048, 512), (1000, 300), (100, 1), (5000, 64), (64, 4096)],   # (L, b)
    [1, 65, 200, 4096],                     # tail + T
    [148, 132, 256, 1],                     # SMs
))


def test_decode_units_stay_within_the_scratch_and_split_bounds(lib):
    tile = lib.dp_tile()
    max_per_split = lib.dp_max_chunks_per_split()
    nc3 = (ctypes.c_int * 3)()
    for B, Hkv, (L, b), tail, sms in SHAPES:
        chunk = lib.dp_decode_chunk(B, Hkv, L, b, tail, sms)
        assert chunk >= tile and chunk % tile == 0, (B, Hkv, L, b, tail, sms, chunk)
        per_head = lib.dp_chunks_per_head(L, b, tail, chunk, nc3)
        full, last, tl = list(nc3)
        n = -(-L // b)
        assert per_head == (n - 1) * full + last + tl
        # every split's keys are covered, by at most kMaxChunksPerSplit units
        assert full * chunk >= min(b, L) and last * chunk >= L - (n - 1) * b and tl * chunk >= tail
        assert max(full, last, tl) <= max_per_split, (B, Hkv, L, b, tail, sms, chunk, nc3[:])
        # the scratch holds every unit, for the tightest capacity L + tail
        units = B * Hkv * per_head
        assert units <= lib.dp_units_bound(B, Hkv, L + tail, b), (B, Hkv, L, b, tail, sms, units)


def test_units_fill_one_wave_when_the_splits_leave_room(lib):
    nc3 = (ctypes.c_int * 3)()
    for B, Hkv, (L, b), tail, sms in SHAPES:
        if sms < 2:
            continue
        n = -(-L // b)
        splits = B * Hkv * (n + 1)
        chunk = lib.dp_decode_chunk(B, Hkv, L, b, tail, sms)
        units = B * Hkv * lib.dp_chunks_per_head(L, b, tail, chunk, nc3)
        if splits <= 2 * sms:
            # one wave of two CTAs per SM, plus one unit per split for its ragged end
            assert units <= 2 * sms + splits, (B, Hkv, L, b, tail, sms, units)
