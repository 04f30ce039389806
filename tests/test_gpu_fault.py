"""The library's failure path on the GPU, made to happen without a fault.

Every pipeline wait in the kernels is bounded: when it runs out it records a
site code in the device fault word and the kernel returns, so the context stays
usable and the host learns of it through w4a16_device_fault().  Here a test
kernel's bounded wait is made to run out (a barrier phase that nothing
completes, a limit of about a millisecond); the site must be reported once,
and the linear layer must work correctly right after it."""
import numpy as np
import pytest
import torch

import oracle
import synth
import weight_only_int4_linear_b200 as w4
from tests._parity import assert_close, bf16_dev_to_f64, bits_to_dev_bf16

pytestmark = pytest.mark.gpu


def _linear_matches_oracle(M, N, K, seed):
    W = synth.weights_f32(seed, synth.TAG_W, N, K)
    pw = w4.PackedWeight.from_float(torch.from_numpy(W).cuda())
    st, qw, sc, z = oracle.quantize_pack(W)
    Xb = synth.activations_bf16(seed + 1, M, K)
    Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(max(w4.workspace_bytes(M, N, K), 256), dtype=torch.uint8, device="cuda")
    w4.linear(bits_to_dev_bf16(Xb), pw.qweight, pw.scales, pw.zeros, Y, ws)
    torch.cuda.synchronize()
    assert int(pw.status.item()) == 0 and st == oracle.OK
    assert_close(bf16_dev_to_f64(Y), oracle.linear(Xb, qw, sc, z), f"M={M} N={N} K={K}")


def test_bounded_wait_reports_its_site_and_the_context_stays_usable(cuda_lib):
    assert w4.device_fault() == 0  # nothing pending from earlier work
    w4.selftest_wait(2_000_000)    # ~1 ms at the SM clock
    assert w4.device_fault() == w4.SELFTEST_SITE
    assert w4.device_fault() == 0  # read and cleared
    for M, N, K in [(1, 300, 1024), (5, 300, 1024), (70, 300, 1024)]:
        _linear_matches_oracle(M, N, K, 40 + M)
    assert w4.device_fault() == 0


def test_first_site_is_kept_until_read(cuda_lib):
    w4.selftest_wait(1_000_000)
    _linear_matches_oracle(1, 256, 512, 77)  # a correct call does not overwrite the recorded site
    w4.selftest_wait(1_000_000)
    assert w4.device_fault() == w4.SELFTEST_SITE
    assert w4.device_fault() == 0


def test_limit_out_of_range_is_rejected_on_the_host(cuda_lib):
    lib = w4.load()
    assert lib.w4a16_selftest_wait(0, None) == w4.ERR_ARG
    assert lib.w4a16_selftest_wait(-5, None) == w4.ERR_ARG
    assert lib.w4a16_selftest_wait(2_000_000_001, None) == w4.ERR_ARG
    assert w4.device_fault() == 0
