"""Shared helpers of the GPU parity tests: the stated tolerance, host<->device
marshalling of BF16 bit patterns, and case setup from the seeded generator."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth

# max |Y - Y_ref| <= 2^-7 |Y_ref| + 1e-3 rms(Y_ref)  and  ||Y - Y_ref||_F / ||Y_ref||_F <= 5e-3
TOL_REL = 2.0 ** -7
TOL_RMS = 1e-3
TOL_FRO = 5e-3
# Y is BF16: below 2^-126 its values are spaced 2^-133 apart, so rounding the output alone can miss a
# relative bound there.  Both bounds carry half that spacing as an absolute term (no effect on outputs
# in the normal range, where it is below 2^-8 of the BF16 spacing).
TOL_ABS_BF16 = 2.0 ** -134


def assert_close(y_gpu: np.ndarray, y_ref: np.ndarray, what: str = "") -> dict:
    """y_gpu: values of the GPU's BF16 outputs (float64); y_ref: oracle FP64 values."""
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    assert y_gpu.shape == y_ref.shape
    assert np.all(np.isfinite(y_gpu)), f"{what}: non-finite outputs"
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    err = np.abs(y_gpu - y_ref)
    bound = TOL_REL * np.abs(y_ref) + TOL_RMS * rms + TOL_ABS_BF16
    bad = err > bound
    # relative Frobenius error, with the output format's absolute resolution taken off the error
    fro_err = max(float(np.linalg.norm(y_gpu - y_ref)) - TOL_ABS_BF16 * np.sqrt(y_ref.size), 0.0)
    fro = fro_err / max(float(np.linalg.norm(y_ref)), 1e-300)
    stats = {"max_err_over_bound": float(np.max(err / np.maximum(bound, 1e-300))), "rel_fro": fro,
             "n": int(y_ref.size)}
    assert not bad.any(), f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; worst index " \
                          f"{np.unravel_index(np.argmax(err - bound), err.shape)} {stats}"
    assert fro <= TOL_FRO, f"{what}: relative Frobenius error {fro}"
    return stats


def bf16_dev_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def bits_to_dev_bf16(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def dev_bf16_to_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def dev_weights(seed: int, tag: int, N: int, K: int) -> torch.Tensor:
    """FP32 weights drawn on the device (bit-identical to synth.weights_f32)."""
    W = torch.empty((N, K), dtype=torch.float32, device="cuda")
    synth.fill_weights_device(seed, tag, W.data_ptr(), N * K, stream=torch.cuda.current_stream().cuda_stream)
    return W


def sample_rows(N: int, count: int, seed: int) -> np.ndarray:
    """Sorted distinct output rows: the first and last 8, plus seeded ones."""
    rng = np.random.default_rng(seed)
    fixed = list(range(min(8, N))) + list(range(max(0, N - 8), N))
    extra = rng.choice(N, size=min(count, N), replace=False)
    return np.unique(np.concatenate([np.array(fixed, dtype=np.int64), extra.astype(np.int64)]))


def oracle_pack_rows(case, rows: np.ndarray):
    """Oracle packing of selected rows of the case's weights (rows are independent)."""
    W = synth.weight_rows_f32(case.w_seed, case.w_tag, case.K, rows)
    st, qw, sc, z = oracle.quantize_pack(W)
    assert st == oracle.OK
    return qw, sc, z
