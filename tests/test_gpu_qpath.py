"""GPU parity of the low-rank query path (csa_q_projection) and the window rows
(csa_window_projection) against the oracle.

The tensor core accumulates in fp32 but not as a sequence of IEEE fp32 additions, so its sums differ
from the float64 ones by an error that scales with the data (bounded here by 1e-4 x RMS), and the
bf16 roundings of qr and of the second product may then land one bf16 step away from the oracle's.
Each stage is therefore checked against the oracle's step applied to the kernel's own input of that
stage (tight), and the final q and window rows also end to end. Values are compared within a bf16-step
bound of their magnitude; in the rotated dims the magnitude is that of the pair, since the rotation
mixes a pair's rounding errors into both outputs."""

import numpy as np
import pytest
import torch

from oracle import csa_oracle as O
from synth.workloads import make_qpath_inputs
from tests.parity import np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops():
    from long_context_decode_c4a_b200 import ops
    return ops


def _rms(a):
    return float(np.sqrt(np.mean(np.asarray(a) ** 2)))


def _bf16_close(got, ref, scale, what):
    """Both sides rounded to bf16: a value near a rounding boundary may go either way, one full bf16
    step (at most 2^-7 relative)."""
    err = np.abs(got - ref)
    bound = 2.0 ** -7 * np.abs(ref) + 1e-4 * scale
    assert np.all(err <= bound), f"{what}: off by more than one bf16 step (worst {np.max(err / bound):.2f})"


def _amplitude(ref, rope_dim=64):
    """|ref|, except in the rotated dims, where an output mixes its pair: there the pair's norm
    (a rounding error of either input reaches both outputs)."""
    amp = np.abs(ref).copy()
    head = ref.shape[-1] - rope_dim
    pair = np.sqrt(ref[..., head::2] ** 2 + ref[..., head + 1::2] ** 2)
    amp[..., head::2] = pair
    amp[..., head + 1::2] = pair
    return amp


def _rel_close(got, ref, rel, absolute, what):
    err = np.abs(got - ref)
    bound = rel * _amplitude(ref) + absolute
    assert np.all(err <= bound), f"{what}: worst {np.max(err / bound):.2f} of the bound"


def _heads_from(qr, wq_b, pos, H, eps=1e-6):
    """The oracle's steps after qr (second product, bf16, per-head norm, RoPE) on a given qr."""
    M = qr.shape[0]
    qraw = O.bf16(qr @ wq_b.T).reshape(M, H, 512)
    q = qraw / np.sqrt(np.mean(qraw * qraw, axis=-1, keepdims=True) + eps)
    return np.stack([O.rope(q[m], float(pos[m]), 64, 10000.0) for m in range(M)])


def _check_q_path(ops, inp, H):
    qa, qr, q = ops.q_projection(inp["x"], inp["wq_a"], inp["gamma_q"], inp["wq_b"], inp["pos"], H=H)
    torch.cuda.synchronize()
    x, wa, wb, g = np64(inp["x"]), np64(inp["wq_a"]), np64(inp["wq_b"]), np64(inp["gamma_q"])
    pos = np64(inp["pos"])
    qa_ref, qr_ref, q_ref = O.q_path(x, wa, g, wb, pos, H)
    qa_g = np64(qa)
    assert np.max(np.abs(qa_g - qa_ref)) <= 1e-4 * _rms(qa_ref), "qa"
    qr_g = np64(qr)
    _bf16_close(qr_g, O.bf16(O.rms_norm(qa_g, g, 1e-6)), 1.0, "qr from the kernel's qa")
    q_g = np64(q)
    # one bf16 step of the second product (2^-7 relative at most) plus the final rounding
    _rel_close(q_g, _heads_from(qr_g, wb, pos, H), 2.0 ** -6, 1e-3, "q vs the oracle's steps on the kernel's qr")
    _rel_close(q_g, q_ref, 2.0 ** -6, 1e-2 * _rms(q_ref), "q end to end")
    return q_g, q_ref


@pytest.mark.parametrize("M", [200, 1, 129])
def test_q_projection_small_shape(ops, M):
    """hidden 512 -> q_rank 256 -> 4 heads x 512: the first product is split over K (two 128-column
    tiles per row tile leave SMs idle) with fp32 reductions; ragged row tiles; positions up to 2^20."""
    inp = make_qpath_inputs(M, hidden=512, q_rank=256, H=4, start_pos=1 << 20, seed=M, device="cuda")
    _check_q_path(ops, inp, 4)


def test_q_projection_pro_decode_shape(ops):
    """64 decode tokens through the Pro query path: hidden 7168 -> 1536 -> 128 heads x 512."""
    inp = make_qpath_inputs(64, start_pos=32767 - 63, seed=3, device="cuda")
    q_g, q_ref = _check_q_path(ops, inp, 128)
    # every head of the kernel's q has unit RMS (rotation keeps the norm)
    assert np.allclose(np.sqrt(np.mean(q_g ** 2, axis=-1)), 1.0, atol=2e-2)


@pytest.mark.parametrize("M,hidden", [(64, 7168), (130, 512)])
def test_window_projection(ops, M, hidden):
    inp = make_qpath_inputs(M, hidden=hidden, q_rank=128, H=1, start_pos=32000, seed=M, device="cuda")
    win = ops.window_projection(inp["x"], inp["wkv"], inp["pos"])
    torch.cuda.synchronize()
    x, wkv, pos = np64(inp["x"]), np64(inp["wkv"]), np64(inp["pos"])
    ref = O.window_projection(x, wkv, pos)
    _rel_close(np64(win), ref, 2.0 ** -6, 1e-2 * _rms(ref), "window rows")


@pytest.mark.parametrize("M,N", [(64, 1024), (64, 256), (130, 1024)])
def test_compressor_stream_projection(ops, M, N):
    """The compressor's kv and score states from the hidden states ([P5] §2.1: [hidden] -> [2 head_dim]
    for the main stream, [2 d_I] for the index stream), rounded to bf16, and the fp32 variant."""
    g = torch.Generator(device="cuda")
    g.manual_seed(M + N)
    x = torch.randn(M, 7168, generator=g, device="cuda").to(torch.bfloat16)
    w = (torch.randn(N, 7168, generator=g, device="cuda") / 84.7).to(torch.bfloat16)
    kv, score = ops.compressor_streams(x, w, w)
    y32 = ops.linear(x, w, torch.float32)
    torch.cuda.synchronize()
    exact = np64(x) @ np64(w).T
    scale = _rms(exact)
    assert np.max(np.abs(np64(y32) - exact)) <= 1e-4 * scale, "fp32 linear"
    # bf16: one bf16 step (kernel and oracle both rounded) plus the accumulation error
    _bf16_close(np64(kv), O.bf16(exact), scale, "kv stream")
    assert torch.equal(kv, score)
