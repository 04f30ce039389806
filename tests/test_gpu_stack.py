"""The 80-layer decode stack (hidden 8192, M = 1, all packed weights resident,
chained on one stream with row renormalisation between layers), checked
teacher-forced: at sampled layers the oracle multiplies sampled weight rows
with the GPU's own BF16 input to that layer, in the same launch sequence the
benchmark times."""
import os
import sys

import numpy as np
import pytest
import torch

import oracle
import synth
import weight_only_int4_linear_b200 as w4
from synth import workloads
from tests._parity import assert_close, bf16_dev_to_f64, dev_bf16_to_bits, oracle_pack_rows, sample_rows

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

pytestmark = pytest.mark.gpu

SAMPLED_LAYERS = (0, 1, 39, 79)


@pytest.fixture(scope="module")
def stack_run(cuda_lib):
    stream = torch.cuda.Stream()
    layers = bench.build_stack(torch, w4, stream)
    buf = bench.StackBuffers(torch, w4, layers)
    c0 = workloads.stack_layer(0)[0]
    x0 = synth.activations_bf16(c0.x_seed, 1, c0.K)
    with torch.cuda.stream(stream):
        buf.h[0].copy_(torch.from_numpy(x0.view(np.int16)).cuda().view(torch.bfloat16))
        h_final, rec = bench.stack_step(w4, layers, buf, record=SAMPLED_LAYERS)
    torch.cuda.synchronize()
    fault = w4.device_fault()
    out = {"x0": x0, "h_final": bf16_dev_to_f64(h_final), "fault": fault,
           "rec": {k: {n: dev_bf16_to_bits(t) for n, t in v.items()} for k, v in rec.items()}}
    del layers, buf
    torch.cuda.empty_cache()
    return out


def test_stack_runs_clean(stack_run):
    assert stack_run["fault"] == 0
    h = stack_run["h_final"]
    assert np.all(np.isfinite(h))
    # the last op is a renorm to unit RMS (BF16 rounding of each element: within 2^-8)
    assert abs(np.sqrt(np.mean(h * h)) - 1.0) < 4e-3
    # the first layer's input is the workload's X itself
    np.testing.assert_array_equal(stack_run["rec"][0]["h"], stack_run["x0"])


@pytest.mark.parametrize("layer", SAMPLED_LAYERS)
def test_stack_layer_teacher_forced(stack_run, layer):
    r = stack_run["rec"][layer]
    inputs = {"qkv": r["h"], "o_proj": r["h"], "gate_up": r["h"], "down": r["u"]}
    for case in workloads.stack_layer(layer):
        name = case.name.split("_", 1)[1]  # "L<layer>_<matrix>"
        rows = sample_rows(case.N, 96, 1000 + layer)
        qw, sc, z = oracle_pack_rows(case, rows)
        ref = oracle.linear(inputs[name], qw, sc, z)
        got = r[name].view(np.uint16)
        got_f = (got.astype(np.uint32) << 16).view(np.float32).astype(np.float64)[:, rows]
        assert_close(got_f, ref, f"stack layer {layer} {name}")


def test_stack_renorm_links(stack_run):
    """u is the renormalised first half of gate+up; both steps use the same kernel the bench runs."""
    for layer in SAMPLED_LAYERS:
        r = stack_run["rec"][layer]
        ref_bits, _ = oracle.renorm(r["gate_up"][:, :bench.STACK_DOWN_IN].copy())
        d = np.abs(r["u"].astype(np.int32) - ref_bits.astype(np.int32))
        assert d.max() <= 1 and np.mean(d != 0) < 1e-3
