"""Shared comparison helpers for the GPU parity tests (CUDA path vs the CPU oracle).

Acceptance rules of the layer specification:
  * compressor output: max abs error <= 5e-3 on the fp32 output; the bf16 output within
    5e-3 plus half a bf16 ulp of the oracle's value;
  * top-k: index sets bit-exact, except where the oracle's k-th and (k+1)-th scores differ
    by less than 1e-3 relative; then they may differ only among entries whose oracle score
    lies within 1e-3 * |k-th score| of the k-th score;
  * attention output: max abs error <= 1e-2 * RMS of the oracle output (fp32 output mode).
"""

from __future__ import annotations

import json
import os

import numpy as np
import torch

from oracle import csa_oracle as O

COMPRESS_ATOL = 5e-3
TOPK_REL = 1e-3
ATTN_REL = 1e-2


def np64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        t = t.detach().to("cpu")
        return t.double().numpy() if t.dtype.is_floating_point else t.numpy()
    return np.asarray(t)


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    """Half of the bf16 spacing at |x| (8 significant bits)."""
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return 0.5 * 2.0 ** (np.floor(np.log2(ax)) - 7)


def assert_compress_close(gpu_f32, gpu_bf16, ref, what=""):
    gpu_f32 = np64(gpu_f32)
    gpu_bf16 = np64(gpu_bf16)
    err = np.max(np.abs(gpu_f32 - ref)) if ref.size else 0.0
    assert err <= COMPRESS_ATOL, f"{what}: fp32 compressor output max abs err {err:.3e} > {COMPRESS_ATOL}"
    tol = COMPRESS_ATOL + bf16_half_ulp(ref)
    bad = np.abs(gpu_bf16 - ref) > tol
    assert not bad.any(), f"{what}: {bad.sum()} bf16 outputs beyond tolerance"


def check_topk(gpu_idx, oracle_scores, k, what=""):
    """READING-17 acceptance of one query's selection; returns the GPU's valid indices."""
    gpu_idx = np.asarray(gpu_idx).astype(np.int64)
    sc = np.asarray(oracle_scores, dtype=np.float64)
    E = sc.shape[0]
    kk = min(k, E)
    valid = gpu_idx[:kk]
    assert np.all(gpu_idx[kk:] == -1), f"{what}: padding must be -1"
    assert np.all((valid >= 0) & (valid < E)), f"{what}: index out of range"
    assert np.all(np.diff(valid) > 0), f"{what}: indices must be strictly ascending"
    if E <= k:
        assert np.array_equal(valid, np.arange(E)), f"{what}: all visible entries must be taken"
        return valid
    ref = O.topk_select(sc, k)[:kk]
    if np.array_equal(ref, valid):
        return valid
    order = np.sort(sc)[::-1]
    sk, sk1 = order[k - 1], order[k]
    assert abs(sk - sk1) < TOPK_REL * abs(sk), (
        f"{what}: selection differs although the k-th/(k+1)-th scores are separated ({sk}, {sk1})")
    band = TOPK_REL * abs(sk)
    must = set(np.nonzero(sc > sk + band)[0].tolist())
    never = set(np.nonzero(sc < sk - band)[0].tolist())
    got = set(valid.tolist())
    assert must <= got, f"{what}: misses {len(must - got)} entries clearly above the k-th score"
    assert not (got & never), f"{what}: selects {len(got & never)} entries clearly below the k-th score"
    return valid


def _log_ratio(what, ratio):
    path = os.environ.get("CSA_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"what": what, "err_over_rms": float(ratio)}) + "\n")


def assert_attn_close(gpu_out, ref, what="", bf16_out=False):
    """fp32 output: max abs error <= 1e-2 * RMS(ref). A bf16 output may in addition differ by half a
    bf16 ulp of the reference value (its own rounding)."""
    gpu_out = np64(gpu_out)
    rms = np.sqrt(np.mean(ref * ref))
    diff = np.abs(gpu_out - ref)
    tol = ATTN_REL * rms + (bf16_half_ulp(ref) if bf16_out else 0.0)
    ratio = float(np.max(diff / tol))
    _log_ratio(what, np.max(diff) / rms)
    if ratio > 1.0:
        d = ref.shape[-1]
        flat = diff.reshape(-1, d)
        h, c = np.unravel_index(np.argmax(flat), flat.shape)
        parts = {"dims[0:256)": flat[:, :256].max(), "dims[256:448)": flat[:, 256:448].max(),
                 "dims[448:512)": flat[:, 448:].max()}
        detail = ", ".join(f"{k} {v:.2e}" for k, v in parts.items())
        raise AssertionError(f"{what}: attention max abs err {np.max(diff):.3e} > tol (1e-2 x RMS {rms:.3e}); "
                             f"worst at head {h} dim {c}; {detail}; worst-head max |ref| {np.abs(ref.reshape(-1, d)[h]).max():.3f}")
    return np.max(diff) / rms
