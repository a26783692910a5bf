"""GPU parity of the grouped output projection (csa_output_projection) against the oracle.

r is bf16: the tensor core accumulates in fp32 but not as a sequence of IEEE fp32 additions, so its
sums differ from the float64 ones by an error that scales with the magnitude of the data (about 1e-5
at K = 4096 here), and r may then land one bf16 step away from the oracle's rounded value: the bound
is one bf16 step of the value plus 1e-4 x RMS(r). y is compared twice: against the oracle's product
of the kernel's own r (isolating the second contraction) and against the oracle's end-to-end y
(1e-2 x RMS, the bar of the attention outputs)."""

import numpy as np
import pytest
import torch

from oracle import csa_oracle as O
from synth.workloads import OPROJ_D, OPROJ_GROUPS, OPROJ_KG, OPROJ_R, make_oproj_inputs
from tests.parity import np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops():
    from long_context_decode_c4a_b200 import ops
    return ops


def _check_r(r_gpu, r_ref, what):
    r_gpu = np64(r_gpu)
    err = np.abs(r_gpu - r_ref)
    bound = 2.0 ** -8 * np.abs(r_ref) + 1e-4 * np.sqrt(np.mean(r_ref ** 2))
    assert np.all(err <= bound), f"{what}: r off by more than one bf16 step (worst {np.max(err / bound):.2f})"


def _check_y(y_gpu, y_from_r, y_ref, what):
    y_gpu = np64(y_gpu)
    scale = np.max(np.abs(y_from_r))
    e1 = np.max(np.abs(y_gpu - y_from_r))
    assert e1 <= 1e-4 * scale, f"{what}: y vs the kernel's r: {e1:.3e} > 1e-4 x {scale:.3e}"
    rms = np.sqrt(np.mean(y_ref ** 2))
    e2 = np.max(np.abs(y_gpu - y_ref))
    assert e2 <= 1e-2 * rms, f"{what}: y vs oracle: {e2:.3e} > 1e-2 x RMS {rms:.3e}"


def _full_check(ops, M, G, Kg, R, D, seed):
    inp = make_oproj_inputs(M, G, Kg, R, D, seed=seed, device="cuda")
    r, y = ops.output_projection(inp["o"], inp["wo_a"], inp["wo_b"])
    torch.cuda.synchronize()
    o, wa, wb = np64(inp["o"]), np64(inp["wo_a"]), np64(inp["wo_b"])
    r_ref, rb_ref, y_ref = O.output_projection(o, wa, wb)
    _check_r(r, r_ref, f"M={M}")
    y_from_r = np64(r) @ wb.T
    _check_y(y, y_from_r, y_ref, f"M={M}")


@pytest.mark.parametrize("M", [200, 1, 128, 129])
def test_output_projection_small_shape(ops, M):
    """G=4 groups of Kg=512 -> R=256, D=384: several N tiles per group, a ragged last M tile, and the
    second product split over K (3 x ceil(M/128) output tiles leave SMs idle) with fp32 reductions."""
    _full_check(ops, M, 4, 512, 256, 384, seed=M)


def test_output_projection_pro_decode_shape(ops):
    """B=64 decode rows through the Pro projection (G=16, Kg=4096, R=1024, D=7168): all of r, and y on
    512 sampled columns."""
    M, G, Kg, R, D = 64, OPROJ_GROUPS, OPROJ_KG, OPROJ_R, OPROJ_D
    inp = make_oproj_inputs(M, seed=5, device="cuda")
    r, y = ops.output_projection(inp["o"], inp["wo_a"], inp["wo_b"])
    torch.cuda.synchronize()
    o = np64(inp["o"])
    r_ref = np.empty((M, G * R))
    for g in range(G):
        r_ref[:, g * R:(g + 1) * R] = o[:, g * Kg:(g + 1) * Kg] @ np64(inp["wo_a"][g]).T
    _check_r(r, r_ref, "pro decode")
    cols = np.sort(np.random.default_rng(0).choice(D, 512, replace=False))
    wb = np64(inp["wo_b"][torch.as_tensor(cols, device="cuda")])
    _check_y(np64(y)[:, cols], np64(r) @ wb.T, O.bf16(r_ref) @ wb.T, "pro decode")


def test_output_projection_prefill_rows_sampled(ops):
    """S=8192 rows through the Pro projection (one output tile per 128 x 128 block, no K split): every
    value of r and y on sampled rows."""
    M, G, Kg, R, D = 8192, OPROJ_GROUPS, OPROJ_KG, OPROJ_R, OPROJ_D
    inp = make_oproj_inputs(M, seed=6, device="cuda")
    r, y = ops.output_projection(inp["o"], inp["wo_a"], inp["wo_b"])
    torch.cuda.synchronize()
    rows = [0, 1, 127, 128, 4095, 6001, 8191]
    o = np64(inp["o"][rows])
    r_ref = np.empty((len(rows), G * R))
    for g in range(G):
        r_ref[:, g * R:(g + 1) * R] = o[:, g * Kg:(g + 1) * Kg] @ np64(inp["wo_a"][g]).T
    rg = np64(r[rows])
    _check_r(rg, r_ref, "prefill rows")
    y_from_r = np.empty((len(rows), D))
    y_ref = np.empty((len(rows), D))
    rb = O.bf16(r_ref)
    for j0 in range(0, D, 1024):
        wb = np64(inp["wo_b"][j0:j0 + 1024])
        y_from_r[:, j0:j0 + 1024] = rg @ wb.T
        y_ref[:, j0:j0 + 1024] = rb @ wb.T
    _check_y(np64(y[rows]), y_from_r, y_ref, "prefill rows")
