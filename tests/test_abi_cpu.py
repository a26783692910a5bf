"""CPU checks of the C ABI: the library loads, exports every symbol include/csa.h declares,
matches the header's struct layouts, and rejects bad arguments on the host before any launch."""

import ctypes
import os
import re
import subprocess
import tempfile

import pytest

from long_context_decode_c4a_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csa.h")


@pytest.fixture(scope="module")
def lib():
    return _lib.load()


def declared_symbols():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^CSA_API\s+[\w\s\*]+?\b((?:csa|hca)_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_symbols()
    for want in ("csa_compress", "csa_indexer_topk", "csa_sparse_attn", "hca_attn", "csa_decode_fused",
                 "hca_decode_fused", "csa_workspace_size", "csa_get_device_status", "csa_state_reset",
                 "csa_output_projection", "csa_q_projection", "csa_window_projection", "csa_indexer_scores",
                 "csa_topk", "csa_linear"):
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\sT\s(\w+)$", out, flags=re.M))
    for name in declared_symbols():
        assert name in exported, name
        assert hasattr(lib, name)
    assert set(_lib.PROTOTYPES) == set(declared_symbols())


def _c_offsets(struct, fields):
    prog = "#include <stdio.h>\n#include <stddef.h>\n#include \"csa.h\"\nint main(void){\n"
    prog += f'printf("%zu\\n", sizeof({struct}));\n'
    for f in fields:
        prog += f'printf("%zu\\n", offsetof({struct}, {f}));\n'
    prog += "return 0;}\n"
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "t.c")
        exe = os.path.join(d, "t")
        open(c, "w").write(prog)
        subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), c, "-o", exe], check=True)
        vals = [int(x) for x in subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split()]
    return vals[0], vals[1:]


@pytest.mark.parametrize("cls,cname", [(_lib.DecodeArgs, "csa_decode_args"), (_lib.HcaDecodeArgs, "hca_decode_args"),
                                       (_lib.CompressorCfg, "csa_compressor_cfg")])
def test_struct_layout_matches_header(cls, cname):
    fields = [f for f, _ in cls._fields_]
    size, offs = _c_offsets(cname, fields)
    assert ctypes.sizeof(cls) == size
    for (f, _), o in zip(cls._fields_, offs):
        assert getattr(cls, f).offset == o, f


def test_status_strings_and_version(lib):
    assert lib.csa_version() == 1
    for code in range(7):
        assert lib.csa_status_string(code)
    assert lib.csa_status_string(99) == b"unknown status"


def test_workspace_sizes(lib):
    n = ctypes.c_size_t()
    assert lib.csa_workspace_size(_lib.CSA_WS_DECODE_FUSED, 64, 1, 8192, 1024, ctypes.byref(n)) == 0
    assert n.value >= 256 + 64 * 8192 * 4 and n.value % 256 == 0
    assert lib.csa_workspace_size(_lib.CSA_WS_INDEXER_TOPK, 8, 1, 262144, 1024, ctypes.byref(n)) == 0
    # long rows need the chunked top-k lists: 16 chunks x 1024 (key, index) pairs per query
    assert n.value >= 256 + 8 * 262144 * 4 + 2 * 8 * 16 * 1024 * 4
    assert lib.csa_workspace_size(_lib.CSA_WS_HCA_ATTN, 64, 1, 256, 0, ctypes.byref(n)) == 0
    assert n.value == 256      # 64 queries: one CTA pair each, no split partials
    # 8 queries: each query's candidates are split over 74 // 8 = 9 CTA pairs, whose partials
    # (O: 128 x 512 fp32, max and denominator: 2 x 128 fp32) live in the workspace
    per_split = (128 * 512 + 2 * 128) * 4
    assert lib.csa_workspace_size(_lib.CSA_WS_SPARSE_ATTN, 8, 1, 262144, 1024, ctypes.byref(n)) == 0
    assert n.value == 256 + 8 * 9 * per_split
    assert lib.csa_workspace_size(_lib.CSA_WS_DECODE_FUSED, 8, 1, 262144, 1024, ctypes.byref(n)) == 0
    assert n.value >= 256 + 8 * 262144 * 4 + 2 * 8 * 16 * 1024 * 4 + 8 * 9 * per_split
    assert lib.csa_workspace_size(_lib.CSA_WS_SPARSE_ATTN, 1, 1, 64, 8, ctypes.byref(n)) == 0
    assert n.value == 256 + 16 * per_split   # at most 16 splits
    assert lib.csa_workspace_size(_lib.CSA_WS_OUTPUT_PROJ, 1, 1, 1, 1, ctypes.byref(n)) == 0
    assert n.value == 256
    assert lib.csa_workspace_size(99, 1, 1, 1, 1, ctypes.byref(n)) == _lib.CSA_ERR_INVALID_ARG
    assert lib.csa_workspace_size(_lib.CSA_WS_DECODE_FUSED, 0, 1, 1, 1, ctypes.byref(n)) == _lib.CSA_ERR_INVALID_ARG


def test_host_side_argument_checks_launch_nothing(lib):
    """Every bad argument is rejected before any CUDA call (this host has no GPU)."""
    cfg = _lib.CompressorCfg(4, 1, 512, 64, 10000.0, 1e-6)
    null = None
    # null pointers
    rc = lib.csa_compress(ctypes.byref(cfg), 1, 4, null, null, null, null, null, null, null, 4096, 8, null, null)
    assert rc == _lib.CSA_ERR_INVALID_ARG
    # unsupported compressor configuration
    bad = _lib.CompressorCfg(8, 1, 512, 64, 10000.0, 1e-6)
    assert lib.csa_compress(ctypes.byref(bad), 1, 4, 16, 16, 16, 16, 16, 16, 16, 4096, 8, null, null) == \
        _lib.CSA_ERR_UNSUPPORTED
    # misaligned pointer (8-byte aligned, not 16)
    assert lib.csa_compress(ctypes.byref(cfg), 1, 4, 16, 24, 16, 16, 16, 16, 16, 4096, 8, null, null) == \
        _lib.CSA_ERR_INVALID_ARG
    # indexer: d_I must be 128, H_I a power of two
    assert lib.csa_indexer_topk(1, 1, 64, 64, 4, 8, 16, 16, 16, 16, 64 * 8, 8, 16, null, 256, 4096, null) == \
        _lib.CSA_ERR_UNSUPPORTED
    assert lib.csa_indexer_topk(1, 1, 48, 128, 4, 8, 16, 16, 16, 16, 128 * 8, 8, 16, null, 256, 4096, null) == \
        _lib.CSA_ERR_UNSUPPORTED
    # indexer: topk over the supported maximum
    assert lib.csa_indexer_topk(1, 1, 64, 128, 4, 4096, 16, 16, 16, 16, 128 * 8, 8, 16, null, 256, 4096, null) == \
        _lib.CSA_ERR_UNSUPPORTED
    # attention: d must be 512, window <= ring_cap, workspace present
    assert lib.csa_sparse_attn(1, 1, 128, 256, 64, 1e4, 0.05, 16, 16, 16, 256 * 128, 128, 128, 16, 256 * 8, 8, 16,
                               8, 16, 16, 0, 256, 256, null) == _lib.CSA_ERR_UNSUPPORTED
    assert lib.csa_sparse_attn(1, 1, 128, 512, 64, 1e4, 0.05, 16, 16, 16, 512 * 64, 64, 128, 16, 512 * 8, 8, 16,
                               8, 16, 16, 0, 256, 256, null) == _lib.CSA_ERR_INVALID_ARG
    assert lib.csa_sparse_attn(1, 1, 128, 512, 64, 1e4, 0.05, 16, 16, 16, 512 * 128, 128, 128, 16, 512 * 8, 8, 16,
                               8, 16, 16, 0, null, 0, null) == _lib.CSA_ERR_WORKSPACE
    # attention: ring stride not a multiple of d
    assert lib.hca_attn(1, 1, 128, 512, 64, 1e4, 0.05, 128, 16, 16, 16, 512 * 128 + 8, 128, 128, 16, 512 * 8, 8, 16,
                        16, 0, 256, 256, null) == _lib.CSA_ERR_INVALID_ARG
    # fused decode: null args
    assert lib.csa_decode_fused(None, null) == _lib.CSA_ERR_INVALID_ARG
    a = _lib.DecodeArgs()
    a.B, a.ratio = 1, 4
    assert lib.csa_decode_fused(ctypes.byref(a), null) in (_lib.CSA_ERR_INVALID_ARG, _lib.CSA_ERR_UNSUPPORTED)
    st = ctypes.c_int()
    assert lib.csa_get_device_status(None, null, ctypes.byref(st)) == _lib.CSA_ERR_INVALID_ARG
    # output projection: null pointers, misalignment, unsupported widths, missing workspace
    assert lib.csa_output_projection(64, 16, 4096, 1024, 7168, null, 16, 16, 16, 16, 256, 256, null) == \
        _lib.CSA_ERR_INVALID_ARG
    assert lib.csa_output_projection(64, 16, 4096, 1024, 7168, 24, 16, 16, 16, 16, 256, 256, null) == \
        _lib.CSA_ERR_INVALID_ARG
    assert lib.csa_output_projection(64, 16, 4000, 1024, 7168, 16, 16, 16, 16, 16, 256, 256, null) == \
        _lib.CSA_ERR_UNSUPPORTED
    assert lib.csa_output_projection(64, 16, 4096, 1000, 7168, 16, 16, 16, 16, 16, 256, 256, null) == \
        _lib.CSA_ERR_UNSUPPORTED
    assert lib.csa_output_projection(64, 16, 4096, 1024, 7168, 16, 16, 16, 16, 16, null, 0, null) == \
        _lib.CSA_ERR_WORKSPACE
    # query path / window rows: d must be 512, q_rank a multiple of 128, pointers present
    assert lib.csa_q_projection(64, 7168, 1536, 128, 256, 64, 1e4, 1e-6, 16, 16, 16, 16, 16, 16, 16, 16, 256, 256,
                                null) == _lib.CSA_ERR_UNSUPPORTED
    assert lib.csa_q_projection(64, 7168, 1500, 128, 512, 64, 1e4, 1e-6, 16, 16, 16, 16, 16, 16, 16, 16, 256, 256,
                                null) == _lib.CSA_ERR_UNSUPPORTED
    assert lib.csa_q_projection(64, 7168, 1536, 128, 512, 64, 1e4, 1e-6, null, 16, 16, 16, 16, 16, 16, 16, 256, 256,
                                null) == _lib.CSA_ERR_INVALID_ARG
    assert lib.csa_window_projection(64, 7168, 512, 63, 1e4, 16, 16, 16, 16, 256, 256, null) == \
        _lib.CSA_ERR_UNSUPPORTED
    assert lib.csa_window_projection(64, 7168, 512, 64, 1e4, 16, 16, 16, 16, null, 0, null) == _lib.CSA_ERR_WORKSPACE
    # the two halves of the indexer: scores required; selection needs scores and a 16-byte aligned row
    assert lib.csa_indexer_scores(1, 1, 64, 128, 4, 16, 16, 16, 16, 128 * 8, 8, null, 256, 256, null) == \
        _lib.CSA_ERR_INVALID_ARG
    assert lib.csa_topk(1, 1, 4, 8, 16, null, 8, 16, 256, 4096, null) == _lib.CSA_ERR_INVALID_ARG
    assert lib.csa_topk(1, 1, 4, 8, 16, 20, 8, 16, 256, 4096, null) == _lib.CSA_ERR_INVALID_ARG
    assert lib.csa_topk(1, 1, 4, 4096, 16, 16, 8, 16, 256, 4096, null) == _lib.CSA_ERR_UNSUPPORTED
    assert lib.csa_linear(64, 1000, 7168, 16, 16, 16, 0, 256, 256, null) == _lib.CSA_ERR_UNSUPPORTED
    assert lib.csa_linear(64, 1024, 7168, null, 16, 16, 0, 256, 256, null) == _lib.CSA_ERR_INVALID_ARG
    assert lib.csa_last_error()


def test_calls_with_no_work_are_refused_before_any_launch(lib):
    """B = 0, S = 0 or M = 0: every entry returns CSA_ERR_INVALID_ARG from its host-side checks (on a
    machine without a GPU, so no CUDA call was reached) and names the size in its error text."""
    cfg = _lib.CompressorCfg(4, 1, 512, 64, 10000.0, 1e-6)
    null, ws = None, 1 << 20
    calls = {
        "compress S=0": lambda: lib.csa_compress(ctypes.byref(cfg), 1, 0, 16, 16, 16, 16, 16, 16, 16, 4096 * 512, 4096,
                                                 null, null),
        "compress B=0": lambda: lib.csa_compress(ctypes.byref(cfg), 0, 4, 16, 16, 16, 16, 16, 16, 16, 4096 * 512, 4096,
                                                 null, null),
        "indexer_topk S=0": lambda: lib.csa_indexer_topk(1, 0, 64, 128, 4, 8, 16, 16, 16, 16, 128 * 8, 8, 16, null,
                                                         256, ws, null),
        "indexer_topk B=0": lambda: lib.csa_indexer_topk(0, 1, 64, 128, 4, 8, 16, 16, 16, 16, 128 * 8, 8, 16, null,
                                                         256, ws, null),
        "indexer_scores S=0": lambda: lib.csa_indexer_scores(1, 0, 64, 128, 4, 16, 16, 16, 16, 128 * 8, 8, 16, 256,
                                                             ws, null),
        "topk S=0": lambda: lib.csa_topk(1, 0, 4, 8, 16, 16, 8, 16, 256, ws, null),
        "sparse_attn S=0": lambda: lib.csa_sparse_attn(1, 0, 128, 512, 64, 1e4, 0.05, 16, 16, 16, 512 * 128, 128, 128,
                                                       16, 512 * 8, 8, 16, 8, 16, 16, 0, 256, ws, null),
        "hca_attn S=0": lambda: lib.hca_attn(1, 0, 128, 512, 64, 1e4, 0.05, 128, 16, 16, 16, 512 * 128, 128, 128, 16,
                                             512 * 8, 8, 16, 16, 0, 256, ws, null),
        "output_projection M=0": lambda: lib.csa_output_projection(0, 16, 4096, 1024, 7168, 16, 16, 16, 16, 16, 256,
                                                                   ws, null),
        "q_projection M=0": lambda: lib.csa_q_projection(0, 7168, 1536, 128, 512, 64, 1e4, 1e-6, 16, 16, 16, 16, 16,
                                                         16, 16, 16, 256, ws, null),
        "window_projection M=0": lambda: lib.csa_window_projection(0, 7168, 512, 64, 1e4, 16, 16, 16, 16, 256, ws,
                                                                   null),
        "linear M=0": lambda: lib.csa_linear(0, 1024, 7168, 16, 16, 16, 0, 256, ws, null),
    }
    for name, call in calls.items():
        assert call() == _lib.CSA_ERR_INVALID_ARG, name
        assert b"positive" in lib.csa_last_error(), name
    n = ctypes.c_size_t()
    for kind in (_lib.CSA_WS_INDEXER_TOPK, _lib.CSA_WS_SPARSE_ATTN, _lib.CSA_WS_HCA_ATTN):
        assert lib.csa_workspace_size(kind, 1, 0, 256, 8, ctypes.byref(n)) == _lib.CSA_ERR_INVALID_ARG



def test_noalloc_refuses_bad_arguments_before_any_cuda_call(lib):
    """The workspace-free indexer checks its arguments first: on this host without a GPU a refused
    call returns the argument error, not the CUDA error that touching its device array would give."""
    p = 1 << 20
    assert lib.csa_indexer_topk_noalloc(1, 1, 64, 128, 4, 8, p, None, p, p, 1024 * 128, 1024, p,
                                        None) == _lib.CSA_ERR_INVALID_ARG
    assert lib.csa_indexer_topk_noalloc(1, 1, 48, 128, 4, 8, p, p, p, p, 1024 * 128, 1024, p,
                                        None) == _lib.CSA_ERR_UNSUPPORTED
    assert lib.csa_indexer_topk_noalloc(1, 1, 64, 128, 4, 4096, p, p, p, p, 1024 * 128, 1024, p,
                                        None) == _lib.CSA_ERR_UNSUPPORTED
    assert lib.csa_indexer_topk_noalloc(0, 1, 64, 128, 4, 8, p, p, p, p, 1024 * 128, 1024, p,
                                        None) == _lib.CSA_ERR_INVALID_ARG
