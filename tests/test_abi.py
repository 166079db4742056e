"""CPU checks of the C-ABI library: it loads, exports every entry point declared in
include/iamap.h, and rejects bad arguments on the host (no GPU needed, no compute call)."""

import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "iamap.h")


@pytest.fixture(scope="module")
def lib():
    from cross_model_attention_map_b200 import build
    build.build()
    from cross_model_attention_map_b200 import iamap
    return iamap


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(iamap_\w+)\s*\(", text)))


def test_header_declares_entry_points():
    names = declared_functions()
    for n in ("iamap_compress", "iamap_compress_stats", "iamap_compress_extract",
              "iamap_mapped_av", "iamap_mapped_av_paged", "iamap_head_match"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (iamap_\w+)", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    raw = ctypes.CDLL(lib.LIB_PATH)
    for n in declared_functions():
        assert hasattr(raw, n)
    # the binding wraps every declared function under the same name
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_plan_counts(lib):
    nrb, ncb, mx = lib.iamap_plan([0, 4096, 12288, 24576, 40960], 4, 64)
    assert (nrb, ncb, mx) == (640, 2080 + 8256 + 18528 + 32896, 256)
    nrb, ncb, mx = lib.iamap_plan([0, 1, 65, 130], 3, 64)
    assert (nrb, ncb, mx) == (1 + 1 + 2, 1 + 1 + 3, 2)


def test_plan_rejects_bad_offsets(lib):
    with pytest.raises(lib.IamapError) as e:
        lib.iamap_plan([0, 10, 5], 2, 64)
    assert e.value.code == -1
    with pytest.raises(lib.IamapError):
        lib.iamap_plan([3, 10], 1, 64)


def test_host_validation_without_gpu(lib):
    """Unsupported block size and null pointers are refused before any device work."""
    raw = lib._lib
    rc = raw.iamap_compress_stats(None, None, None, None, 1, 64, 8, 64, 32, 0.9, 0, 0.0, None,
                                  None, None, None, None, None, None, None, None, 0, None)
    assert rc == -2 and "B = 64" in lib.iamap_last_error()
    rc = raw.iamap_compress_stats(None, None, None, None, 1, 64, 8, 64, 64, 0.9, 0, 0.0, None,
                                  None, None, None, None, None, None, None, None, 0, None)
    assert rc == -1
    rc = raw.iamap_mapped_av_paged(None, 0, None, None, 0, None, 0, 16, None, None, 1, 1, 1, 8,
                                   None, None, 0, None)
    assert rc == -1
    rc = raw.iamap_head_match(None, None, 1, 1, 64, None, None, 1, 1, 128, 8, 8, None, None, None,
                              0, None)
    assert rc == -1
    st = ctypes.c_int(0)
    assert raw.iamap_device_status(None, None) == -1


def test_workspace_queries(lib):
    assert lib.iamap_compress_workspace_bytes(4, 640) > 640 * 8
    assert lib.iamap_head_match_workspace_bytes(24, 14, 8, 64, 1024) > 848 * 136 * 8192
    assert lib.iamap_mapped_av_paged_workspace_bytes(4, 64, 128, 8704, 16) > 0


def test_host_validation_of_variants(lib):
    """The metric, grouped-value, consistency and self-test entry points refuse bad arguments
    on the host."""
    raw = lib._lib
    rc = raw.iamap_head_match_metric(None, None, 1, 1, 64, None, None, 1, 1, 128, 8, 8, 7, None,
                                     None, None, 0, None)
    assert rc == -1 and "metric" in lib.iamap_last_error()
    rc = raw.iamap_mapped_av_gqa(None, None, 1, 64, 64, 4, None, None, None, None, None, 0, None,
                                 8, 3, None, 64, None, None, 0, None)
    assert rc == -1 and "divide" in lib.iamap_last_error()
    rc = raw.iamap_mapped_av_paged_gqa(None, 0, None, None, 0, None, 0, 16, None, None, 1, 1, 8,
                                       3, 64, None, None, 0, None)
    assert rc == -1 and "divide" in lib.iamap_last_error()
    assert raw.iamap_mapping_consistency(None, None, 4, None, None) == -1
    assert raw.iamap_selftest_wait_timeout(0, None, None) == -1
    assert raw.iamap_selftest_wait_timeout(2_000_000, None, None) == -1


def test_host_validation_of_prefix_index(lib):
    """The prefix-index entry points refuse bad arguments on the host and count keys there."""
    raw = lib._lib
    assert lib.iamap_prefix_num_keys([0, 64, 100, 100, 300], 4, 64) == 4
    assert lib.iamap_prefix_num_keys([5, 5], 1, 1) == 0
    n = ctypes.c_int64(0)
    cu = (ctypes.c_int32 * 3)(0, 10, 4)
    assert raw.iamap_prefix_num_keys(cu, 2, 4, ctypes.byref(n)) == -1   # decreasing offsets
    assert raw.iamap_prefix_num_keys(cu, 2, 0, ctypes.byref(n)) == -1   # B < 1
    fake = 256   # never dereferenced: every call below fails validation first
    # block size outside [1, 4096]
    assert raw.iamap_prefix_keys(fake, 64, fake, 1, 0, 0, fake, 1, fake, None) == -1
    assert raw.iamap_prefix_keys(fake, 64, fake, 1, 4097, 0, fake, 1, fake, None) == -1
    # null key_cu / null keys with a positive capacity / null tokens with n > 0
    assert raw.iamap_prefix_keys(fake, 64, fake, 1, 64, 0, fake, 1, None, None) == -1
    assert raw.iamap_prefix_keys(fake, 64, fake, 1, 64, 0, None, 1, fake, None) == -1
    assert raw.iamap_prefix_keys(None, 64, fake, 1, 64, 0, fake, 1, fake, None) == -1
    # capacity not a power of two, or out of range
    for cap in (0, 3, 100, 1 << 41):
        assert raw.iamap_prefix_index_clear(fake, fake, cap, None) == -1
        assert raw.iamap_prefix_insert(fake, fake, 1, fake, fake, cap, fake, None) == -1
        assert raw.iamap_prefix_lookup(fake, 1, None, 0, fake, fake, cap, fake, None, None) == -1
    assert "power of two" in lib.iamap_last_error()
    # null table, null outputs, negative counts, key_cu without hit_blocks
    assert raw.iamap_prefix_insert(fake, fake, 1, None, fake, 16, fake, None) == -1
    assert raw.iamap_prefix_insert(fake, fake, 1, fake, fake, 16, None, None) == -1
    assert raw.iamap_prefix_insert(fake, fake, -1, fake, fake, 16, fake, None) == -1
    assert raw.iamap_prefix_lookup(fake, 1, fake, 1, fake, fake, 16, fake, None, None) == -1
    assert "together" in lib.iamap_last_error()
    assert raw.iamap_prefix_lookup(fake, 1, fake, 0, fake, fake, 16, fake, fake, None) == -1
    assert raw.iamap_prefix_lookup(None, 1, None, 0, fake, fake, 16, fake, None, None) == -1


def _prototypes():
    """name -> number of parameters of every prototype in the header."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for m in re.finditer(r"\b(?:int|size_t|const char\s*\*)\s+(iamap_\w+)\s*\(([^)]*)\)\s*;",
                         text):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else len(params.split(","))
    return out


def test_binding_signatures_match_header(lib):
    """Every ctypes signature of the binding has the header prototype's parameter count, and
    every header prototype has a signature."""
    protos = _prototypes()
    assert len(protos) >= 24
    sigs = lib._SIGS
    assert sorted(protos) == sorted(sigs)
    for name, count in protos.items():
        assert len(sigs[name][1]) == count, name


def test_header_compiles_as_c_and_links(lib, tmp_path):
    """A plain C99 program includes iamap.h, links libiamap.so and calls host-only entry points
    (planning and argument checks; no device work)."""
    src = tmp_path / "abi.c"
    src.write_text(r'''
#include <stdio.h>
#include "iamap.h"
int main(void) {
  int32_t cu[4] = {0, 64, 100, 300};
  int64_t rb = 0, cbk = 0, nk = 0;
  int32_t mx = 0;
  if (iamap_plan(cu, 3, 64, &rb, &cbk, &mx) != IAMAP_OK) return 1;
  if (rb != 6 || cbk != 1 + 1 + 10 || mx != 4) return 2;
  if (iamap_prefix_num_keys(cu, 3, 64, &nk) != IAMAP_OK || nk != 1 + 0 + 3) return 3;
  if (iamap_prefix_insert(NULL, NULL, 1, NULL, NULL, 3, NULL, NULL) != IAMAP_ERR_INVALID_ARG)
    return 4;
  if (iamap_last_error()[0] == 0) return 5;
  if (iamap_version() < 1) return 6;
  printf("ok %lld %lld %d %lld\n", (long long)rb, (long long)cbk, mx, (long long)nk);
  return 0;
}
''')
    exe = tmp_path / "abi"
    libdir = os.path.dirname(lib.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), "-L", libdir, "-liamap",
                    "-Wl,-rpath," + libdir], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, (out.returncode, out.stdout, out.stderr)
    assert out.stdout.startswith("ok 6 12 4 4")


def test_chunk_plan_counts_and_checks(lib):
    """Chunk plan on the host: only the chunks' row blocks and causal blocks are counted; starts
    that are not multiples of B, or chunks that do not end at their key length, are refused."""
    # sequence 0: keys 228 (4 blocks), chunk from 128 (blocks 2, 3); sequence 1: keys 192
    # (3 blocks), chunk from 128 (block 2)
    assert lib.iamap_chunk_plan([0, 100, 164], [0, 228, 420], [128, 128], 2, 64) == (3, 7 + 3, 4)
    # whole sequences as chunks: the plan of the sequences themselves
    assert lib.iamap_chunk_plan([0, 4096, 12288], [0, 4096, 12288], [0, 0], 2, 64) == \
        lib.iamap_plan([0, 4096, 12288], 2, 64)
    # a chunk at the end of a sequence that holds no rows
    assert lib.iamap_chunk_plan([0, 0], [0, 128], [128], 1, 64) == (0, 0, 2)
    with pytest.raises(lib.IamapError) as e:
        lib.iamap_chunk_plan([0, 200], [0, 300], [100], 1, 64)       # 100 is not a multiple of 64
    assert e.value.code == -1 and "multiple" in lib.iamap_last_error()
    with pytest.raises(lib.IamapError) as e:
        lib.iamap_chunk_plan([0, 100], [0, 300], [128], 1, 64)       # ends at 228, keys 300
    assert e.value.code == -1


def test_host_validation_of_chunk_and_sender_output(lib):
    """The chunk and sender-output entry points refuse bad arguments before any device work."""
    raw = lib._lib
    fake = 256   # never dereferenced: every call below fails validation first
    # d_vs must be 64 or 128
    rc = raw.iamap_compress_with_output(fake, fake, fake, None, 1, 64, 4, 64, 64, 0.9, 0, 0.0,
                                        fake, 96, fake, fake, fake, fake, fake, fake, fake, fake,
                                        fake, fake, 1, fake, 0, None)
    assert rc == -2 and "d_vs" in lib.iamap_last_error()
    # v_s without o_s
    rc = raw.iamap_compress_chunk(fake, fake, fake, fake, fake, None, None, None, 1, 64, 64, 4, 64,
                                  64, 0.9, 0, 0.0, fake, 64, None, fake, fake, fake, fake, fake,
                                  fake, fake, fake, fake, 1, fake, 0, None)
    assert rc == -1 and "together" in lib.iamap_last_error()
    # grouped values must divide the receiver heads
    rc = raw.iamap_mapped_av_chunk(fake, fake, fake, None, None, None, 1, 64, 64, 64, 4, fake,
                                   fake, fake, fake, fake, 1, fake, 8, 3, fake, 64, fake, fake, 0,
                                   None)
    assert rc == -1 and "divide" in lib.iamap_last_error()


def test_layers_plan_counts(lib):
    """Several layers per launch: the stacked batch has num_layers copies of every sequence."""
    one = lib.iamap_plan([0, 300, 370, 371], 3, 64)
    assert lib.iamap_layers_plan([0, 300, 370, 371], 3, 4, 64) == (4 * one[0], 4 * one[1], one[2])
    with pytest.raises(lib.IamapError):
        lib.iamap_layers_plan([0, 300], 1, 0, 64)
    assert lib.iamap_layers_workspace_bytes(3, 4, 4 * one[0]) > \
        lib.iamap_compress_workspace_bytes(12, 4 * one[0])
