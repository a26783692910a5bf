"""The workspace-free indexer + top-k entry point (csa_indexer_topk_noalloc).

It serves callers that cannot allocate device memory where they run the layer (code inside
another framework's memory pool, plugins handed only their input and output tensors, paths that
must never call cudaMalloc): its scratch lives in a fixed array that the library defines in device
memory. This file is collected last so that a failure here leaves every other test already run;
it passes both alone in a fresh process and after the rest of the suite.
"""

import math

import pytest
import torch

pytestmark = pytest.mark.gpu


def _inputs(seed, B, S, H_I, E):
    g = torch.Generator().manual_seed(seed)
    q_idx = torch.randn(B, S, H_I, 128, generator=g).to(torch.bfloat16).cuda()
    w = (torch.randn(B, S, H_I, generator=g) / math.sqrt(128) / math.sqrt(H_I)).cuda()
    cache = torch.randn(B, E, 128, generator=g).to(torch.bfloat16).cuda()
    pos = torch.full((B, S), 4 * E - 1, dtype=torch.int32)
    pos[:, 0] -= 4 * (seed % 7)     # a few requests see fewer entries
    return pos.cuda(), q_idx, w, cache


def _noalloc(lib, pos, q_idx, w, cache, topk):
    B, S, H_I, d_I = q_idx.shape
    out = torch.full((B, S, topk), -7, dtype=torch.int32, device="cuda")
    rc = lib.csa_indexer_topk_noalloc(B, S, H_I, d_I, 4, topk, pos.data_ptr(), q_idx.data_ptr(), w.data_ptr(),
                                      cache.data_ptr(), cache.stride(0), cache.shape[1], out.data_ptr(),
                                      torch.cuda.current_stream().cuda_stream)
    assert rc == 0, lib.csa_status_string(rc)
    return out


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    from long_context_decode_c4a_b200 import _lib, ops
    lib = _lib.load()
    for call, (seed, B, S, E, topk) in enumerate(((1, 8, 1, 8192, 1024), (2, 4, 3, 4000, 256))):
        pos, q_idx, w, cache = _inputs(seed, B, S, 64, E)
        got = _noalloc(lib, pos, q_idx, w, cache, topk)
        ref = ops.indexer_topk(pos, q_idx, w, cache, topk)
        torch.cuda.synchronize()
        assert torch.equal(got, ref), f"call {call}: selection differs from csa_indexer_topk"


def test_noalloc_refuses_sizes_beyond_its_array():
    from long_context_decode_c4a_b200 import _lib
    lib = _lib.load()
    # Nothing is launched for a refused call, so aligned stand-in addresses serve as the tensors.
    p = 1 << 20
    # 65 queries x 16384 entries of fp32 scores exceed the 4 MiB array; 16385 entries exceed one chunk.
    assert lib.csa_indexer_topk_noalloc(65, 1, 64, 128, 4, 8, p, p, p, p, 16384 * 128, 16384, p,
                                        None) == _lib.CSA_ERR_UNSUPPORTED
    assert lib.csa_indexer_topk_noalloc(1, 1, 64, 128, 4, 8, p, p, p, p, 16385 * 128, 16385, p,
                                        None) == _lib.CSA_ERR_UNSUPPORTED
    # Arguments csa_indexer_topk refuses are refused here too, before the array is written.
    assert lib.csa_indexer_topk_noalloc(1, 1, 48, 128, 4, 8, p, p, p, p, 1024 * 128, 1024, p,
                                        None) == _lib.CSA_ERR_UNSUPPORTED
    assert lib.csa_indexer_topk_noalloc(1, 1, 64, 128, 4, 8, p, None, p, p, 1024 * 128, 1024, p,
                                        None) == _lib.CSA_ERR_INVALID_ARG
