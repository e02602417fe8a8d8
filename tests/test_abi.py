"""Host-only checks of the C-ABI library: it builds, loads, exports every
symbol ``include/dsa.h`` declares, and rejects bad arguments on the host
before touching the GPU (no compute call is made here)."""
import ctypes
import os
import re
import subprocess

import pytest

from long_context_fp8_b200 import build as dsa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dsa.h")


@pytest.fixture(scope="module")
def lib():
    dsa_build.build()
    from long_context_fp8_b200 import dsa
    return dsa.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"\b(dsa_[a-z_0-9]+)\s*\(", src)
    return sorted(set(names))


def test_header_and_binding_agree():
    from long_context_fp8_b200 import dsa
    assert sorted(dsa.EXPORTS) == declared_functions()


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", dsa_build.LIB], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(dsa_\w+)", out))
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(lib, name)


def test_version_and_status_strings(lib):
    assert lib.dsa_version() == (0 << 16) | 1
    assert lib.dsa_status_string(0) == b"DSA_OK"
    assert lib.dsa_status_string(5) == b"DSA_ERR_TIMEOUT"
    assert lib.dsa_status_string(99) == b"DSA_ERR_UNKNOWN"


def test_workspace_sizes(lib):
    assert lib.dsa_topk_workspace_size(10, 100, 8) == 0
    T, k = 131072, 2048
    ws = lib.dsa_prefill_workspace_size(T, 64, 128, 128, 128, k, 2)
    assert ws >= 256 + T * k * 4 + 64 * T * 4
    assert ws % 256 == 0
    assert lib.dsa_prefill_workspace_size(0, 64, 128, 128, 128, k, 2) == 0
    wd = lib.dsa_decode_workspace_size(64, 65536, 128, 128, 2048)
    assert wd >= 256 + 64 * 65536 * 4 + 64 * 2048 * 4


def test_host_argument_errors(lib):
    P = ctypes.c_void_p
    fake = P(0x1000)            # never dereferenced: every call below fails validation first
    INVALID, UNSUP, WS = 1, 2, 3
    # null pointers
    assert lib.dsa_index_scores(None, None, None, None, None, 10, 4, 64, 0, 1, fake, 10, 1, 0, None) == INVALID
    # fp32 indexer must not get scales
    assert lib.dsa_index_scores(fake, fake, fake, fake, fake, 10, 4, 64, 0, 1, fake, 10, 1, 0, None) == INVALID
    # unsupported fp8 head dim
    assert lib.dsa_index_scores(fake, fake, fake, fake, fake, 10, 4, 64, 0, 1, fake, 10, 1, 2, None) == UNSUP
    # row range out of bounds / short leading dimension
    assert lib.dsa_index_scores(fake, None, fake, None, fake, 10, 4, 64, 5, 6, fake, 10, 1, 0, None) == INVALID
    assert lib.dsa_index_scores(fake, None, fake, None, fake, 10, 4, 64, 0, 6, fake, 9, 1, 0, None) == INVALID
    # misaligned pointer
    assert lib.dsa_index_scores(P(0x1001), None, fake, None, fake, 10, 4, 64, 0, 1, fake, 10, 1, 0, None) == INVALID
    # top-k: bad k, bad rows
    assert lib.dsa_topk(fake, 10, 0, 1, 10, 0, fake, None, 0, None) == INVALID
    assert lib.dsa_topk(fake, 10, 0, 1, 10, 70000, fake, None, 0, None) == INVALID
    assert lib.dsa_topk(fake, 10, 8, 3, 10, 4, fake, None, 0, None) == INVALID
    # attention: unsupported head dim, bad k
    assert lib.dsa_sparse_attn(fake, fake, fake, fake, 10, 4, 96, 8, 1.0, fake, None, 1, None) == UNSUP
    assert lib.dsa_sparse_attn(fake, fake, fake, fake, 10, 4, 64, 0, 1.0, fake, None, 1, None) == INVALID
    assert lib.dsa_sparse_attn(fake, fake, fake, fake, 10, 200, 128, 8, 1.0, fake, None, 1, None) == UNSUP
    assert lib.dsa_sparse_attn(fake, fake, fake, fake, 10, 4, 64, 8, float("nan"), fake, None, 1, None) == INVALID
    # prefill: missing / short / misaligned workspace
    args = [fake, fake, fake, fake, fake, fake, fake, fake, 1000, 64, 128, 16, 128, 64, 0.1, fake,
            None, None, 2]
    assert lib.dsa_prefill(*args, None, 0, None) == WS
    assert lib.dsa_prefill(*args, fake, 1024, None) == WS
    assert lib.dsa_prefill(*args, P(0x1080), 1 << 30, None) == WS
    # host-memory prefill: E4M3 only, null host pointer, missing / short workspace
    hws = lib.dsa_prefill_host_workspace_size(1000, 64, 128, 16, 128, 64, 2)
    assert hws > 1000 * (64 * 128 + 2 * 16 * 128 * 2)          # at least q_idx, q and out mirrors
    assert lib.dsa_prefill_host_workspace_size(1000, 64, 128, 16, 128, 64, 0) == 0
    assert lib.dsa_prefill_host(*args[:-1], 0, fake, hws, None) == UNSUP
    bad = list(args)
    bad[5] = None                                                # q
    assert lib.dsa_prefill_host(*bad, fake, hws, None) == INVALID
    assert lib.dsa_prefill_host(*args, None, hws, None) == WS
    assert lib.dsa_prefill_host(*args, fake, hws - 256, None) == WS
    # decode: unsupported page size, short workspace
    dargs = [fake] * 10 + [100, 4, 64, 2, 256, 64, 128, 128, 128, 64, 0.1, fake, None, None]
    assert lib.dsa_decode(*dargs, fake, 10, None) == WS
    dargs_bad = list(dargs)
    dargs_bad[12] = 24          # page_size not a multiple of 16
    assert lib.dsa_decode(*dargs_bad, fake, 1 << 30, None) == UNSUP
    assert lib.dsa_stream_status(None, None) == INVALID


def test_host_argument_errors_window_quantiser_kv8(lib):
    """The sliding-window, quantiser, cache-append and FP8 K/V entry points
    reject bad arguments on the host, before any launch (no GPU needed)."""
    P = ctypes.c_void_p
    fake = P(0x1000)            # never dereferenced: every call below fails validation first
    OK, INVALID, UNSUP, WS = 0, 1, 2, 3
    # window top-k: negative / too large window, bad k, rows out of range; no rows is a no-op
    assert lib.dsa_topk_window(fake, 10, 0, 1, 10, 4, -1, fake, None, 0, None) == INVALID
    assert lib.dsa_topk_window(fake, 10, 0, 1, 10, 4, (1 << 24) + 1, fake, None, 0, None) == INVALID
    assert lib.dsa_topk_window(fake, 10, 0, 1, 10, 0, 8, fake, None, 0, None) == INVALID
    assert lib.dsa_topk_window(fake, 10, 8, 3, 10, 4, 8, fake, None, 0, None) == INVALID
    assert lib.dsa_topk_window(fake, 10, 0, 0, 10, 4, 8, fake, None, 0, None) == OK
    # prefill / decode with a window: negative window
    pargs = [fake] * 8 + [1000, 64, 128, 16, 128, 64, -1, 0.1, fake, None, None, 2, fake, 1 << 30, None]
    assert lib.dsa_prefill_window(*pargs) == INVALID
    dargs = [fake] * 10 + [100, 4, 64, 2, 256, 64, 128, 128, 128, 64, -1, 0.1, fake, None, None, fake, 1 << 30, None]
    assert lib.dsa_decode_window(*dargs) == INVALID
    # FP8 K/V decode: scales required; heads the tensor-core attention cannot take
    kargs = [fake] * 6 + [fake, None, fake, fake] + [fake, fake, 100, 4, 64, 2, 256, 64, 128, 128, 128, 64, 0,
                                                      0.1, fake, None, None, fake, 1 << 30, None]
    assert lib.dsa_decode_kv8(*kargs) == INVALID
    kargs[7] = fake
    kargs[19] = 16                                               # H_q
    assert lib.dsa_decode_kv8(*kargs) == UNSUP
    kargs[19] = 128
    kargs[18] = 64                                               # d_I
    assert lib.dsa_decode_kv8(*kargs) == UNSUP
    # quantiser: dtype, width, alignment; no rows is a no-op
    assert lib.dsa_quantize_e4m3(fake, 2, 4, 128, fake, fake, None) == UNSUP         # E4M3 input
    assert lib.dsa_quantize_e4m3(fake, 1, 4, 12, fake, fake, None) == UNSUP          # cols % 8
    assert lib.dsa_quantize_e4m3(fake, 1, 4, 16392, fake, fake, None) == UNSUP       # cols > 16384
    assert lib.dsa_quantize_e4m3(fake, 1, 4, 128, P(0x1004), fake, None) == INVALID  # codes not 8-aligned
    assert lib.dsa_quantize_e4m3(P(0x1008), 1, 4, 128, fake, fake, None) == INVALID  # x not 16-aligned
    assert lib.dsa_quantize_e4m3(None, 1, 4, 128, fake, fake, None) == INVALID
    assert lib.dsa_quantize_e4m3(fake, 1, 0, 128, fake, fake, None) == OK
    # cache append: nothing to do, null pointers, key width, status alignment, dtype
    aargs = [fake, 1, fake, fake, fake, fake, 5, 2, fake, 4, 100, 64, 128, 128, fake, fake, fake, fake, None, None]
    assert lib.dsa_cache_append(*aargs[:6], 0, *aargs[7:]) == OK
    bad = list(aargs); bad[2] = None
    assert lib.dsa_cache_append(*bad) == INVALID
    bad = list(aargs); bad[12] = 264                             # d_I
    assert lib.dsa_cache_append(*bad) == UNSUP
    bad = list(aargs); bad[18] = P(0x1002)                       # status
    assert lib.dsa_cache_append(*bad) == INVALID
    bad = list(aargs); bad[1] = 2                                # E4M3 keys
    assert lib.dsa_cache_append(*bad) == UNSUP
    # FP8 K/V append: the K/V scale caches are required; d up to 256
    kv = [fake, 1, fake, fake, fake, fake, 5, 2, fake, 4, 100, 64, 128, 128, fake, fake, fake, None, fake, fake,
          None, None]
    assert lib.dsa_cache_append_kv8(*kv) == INVALID
    kv[17] = fake
    kv[13] = 264                                                 # d
    assert lib.dsa_cache_append_kv8(*kv) == UNSUP


def test_host_argument_errors_split_decode(lib):
    """The split-context entry points reject bad arguments on the host, before
    any launch (no GPU needed)."""
    P = ctypes.c_void_p
    fake = P(0x1000)            # never dereferenced: every call below fails validation first
    OK, INVALID, UNSUP, WS = 0, 1, 2, 3
    ws = lib.dsa_split_workspace_size(8, 4, 131072, 128, 128, 512)
    assert ws >= 256 + 4 * 131072 * 4 + 8 * 4 * 512 * 4
    assert lib.dsa_split_workspace_size(0, 4, 131072, 128, 128, 512) == 0
    # select: pos_base required; index shape; workspace size
    sargs = [fake] * 8 + [100, 4, 64, 2, 256, 64, 128, 64, fake, fake, fake, 1 << 30, None]
    bad = list(sargs); bad[7] = None
    assert lib.dsa_decode_select(*bad) == INVALID
    bad = list(sargs); bad[14] = 64                              # d_I
    assert lib.dsa_decode_select(*bad) == UNSUP
    bad = list(sargs); bad[15] = 0                               # k_sel
    assert lib.dsa_decode_select(*bad) == INVALID
    bad = list(sargs); bad[19] = 16                              # ws_bytes
    assert lib.dsa_decode_select(*bad) == WS
    # merge of selections: sizes, a list stride shorter than a list
    assert lib.dsa_merge_selections(fake, fake, 0, 0, 4, 64, fake, fake, 1 << 30, None) == INVALID
    assert lib.dsa_merge_selections(fake, fake, 100, 2, 4, 64, fake, fake, 1 << 30, None) == INVALID
    assert lib.dsa_merge_selections(fake, fake, 0, 2, 4, 64, fake, fake, 16, None) == WS
    # attend: lse required; one FP8 scale without the other; d
    aargs = [fake, fake, None, fake, None, fake, fake, fake, 100, 4, 64, 2, 128, 128, 64, fake, 0.1, fake, fake,
             fake, 1 << 30, None]
    bad = list(aargs); bad[18] = None
    assert lib.dsa_decode_attend(*bad) == INVALID
    bad = list(aargs); bad[2] = fake
    assert lib.dsa_decode_attend(*bad) == INVALID
    bad = list(aargs); bad[13] = 64                              # d
    assert lib.dsa_decode_attend(*bad) == UNSUP
    # merge of partials: d, strides, alignment
    assert lib.dsa_merge_partials(fake, 0, fake, 0, 2, 4, 128, 64, fake, None, None) == UNSUP
    assert lib.dsa_merge_partials(fake, 100, fake, 0, 2, 4, 128, 128, fake, None, None) == INVALID
    assert lib.dsa_merge_partials(fake, 0, P(0x1002), 0, 2, 4, 128, 128, fake, None, None) == INVALID
    assert lib.dsa_merge_partials(fake, 65540, fake, 0, 2, 4, 128, 128, fake, None, None) == INVALID


def test_header_compiles_as_c_and_library_links(lib, tmp_path):
    """A C99 program that includes include/dsa.h, links the shared library and
    calls the entry points that need no GPU."""
    exe = str(tmp_path / "abi_consumer")
    src = os.path.join(ROOT, "tests", "abi_consumer.c")
    libdir = os.path.dirname(dsa_build.LIB)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"), src,
                    "-o", exe, f"-L{libdir}", "-l:libdsa_b200.so", f"-Wl,-rpath,{libdir}"], check=True,
                   capture_output=True, text=True)
    r = subprocess.run([exe], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)


def test_prefill_workspace_is_linear_in_the_sequence_length(lib):
    """The fused selection keeps no T x T score matrix: beyond the selection
    itself (T x k indices) the workspace stays within a fixed budget, so it
    grows linearly with T instead of quadratically."""
    from long_context_fp8_b200 import dsa
    k = 2048
    sizes = {T: lib.dsa_prefill_workspace_size(T, 64, 128, 128, 128, k, dsa.DSA_E4M3)
             for T in (1 << 17, 1 << 18, 1 << 19)}
    for T, size in sizes.items():
        assert size - T * k * 4 < (3 << 29), (T, size)     # under 1.5 GiB besides the indices
    assert sizes[1 << 18] < 2.2 * sizes[1 << 17]
    assert sizes[1 << 19] < 2.2 * sizes[1 << 18]
