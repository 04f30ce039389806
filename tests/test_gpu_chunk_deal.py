"""The one-token GEMV deals out its work in chunks of 2 or 4 quantisation groups of a 128-row tile, taken
from a counter in the workspace, and a dependent kernel adds each tile's chunk sums in slot order (two
parts per row over whole tiles, or four over half tiles where a tile has more than 64 chunks).

Checked here: outputs against the FP64 oracle for both chunk sizes (4 where every CTA streams 12 or more
units, else 2) and ragged last row tiles; the same bits on every call whichever
CTAs took which chunks; and the counter area back at zero after every call, so that calls of other
shapes sharing the workspace see it as they must."""
import numpy as np
import pytest
import torch

import oracle
import synth
import weight_only_int4_linear_b200 as w4
from tests._parity import assert_close, bf16_dev_to_f64, bits_to_dev_bf16, dev_weights, sample_rows

pytestmark = pytest.mark.gpu

COUNTER_BYTES = 256 * 1024


def _packed(N, K, seed):
    W = dev_weights(seed, synth.TAG_W, N, K)
    pw = w4.PackedWeight.from_float(W)
    torch.cuda.synchronize()
    assert int(pw.status.item()) == 0
    return pw


def _oracle_rows(N, K, seed, X, rows):
    W = synth.weight_rows_f32(seed, synth.TAG_W, K, rows)
    st, qw, sc, z = oracle.quantize_pack(W)
    assert st == oracle.OK
    return oracle.linear(X, qw, sc, z)


@pytest.mark.parametrize("N,K", [(300, 1024),     # 3 row tiles, the last of 44 rows; 8 groups per row
                                 (129, 1024),     # a one-row last tile
                                 (4096, 4096),    # 1024 units: chunks of 2
                                 (8192, 16384),   # 8192 units: chunks of 4 on a 148-SM part
                                 (300, 32768)])   # 128 chunks per tile: the reduction's four parts per row
                                                  # over half tiles, the last half tile past N
def test_chunked_one_token_gemv(cuda_lib, N, K):
    seed = 7 + N + K
    pw = _packed(N, K, seed)
    X = synth.activations_bf16(seed, 1, K)
    Xd = bits_to_dev_bf16(X)
    nbytes = w4.workspace_bytes(1, N, K)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(3):
        Y = torch.full((1, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        w4.linear(Xd, pw.qweight, pw.scales, pw.zeros, Y, ws, path=w4.PATH_DECODE)
        outs.append(Y)
    torch.cuda.synchronize()
    assert not ws[:COUNTER_BYTES].any().item()  # the chunk counter and row counters back at zero
    for Y in outs[1:]:
        assert torch.equal(Y.view(torch.int16), outs[0].view(torch.int16))
    rows = np.arange(N) if N <= 512 else sample_rows(N, 256, seed)
    ref = _oracle_rows(N, K, seed, X, rows)
    got = bf16_dev_to_f64(outs[0])[:, rows]
    assert_close(got, ref, f"N={N} K={K}")
    assert np.all(np.isfinite(bf16_dev_to_f64(outs[0])))


def test_interleaved_shapes_share_the_counter(cuda_lib):
    """Calls of three shapes, in turn, on one workspace zeroed once: each call must find the chunk counter
    at zero (or it would skip chunks) and leave it there."""
    shapes = [(1000, 2048), (5120, 5120), (130, 1024)]
    packs = [_packed(N, K, 11 + i) for i, (N, K) in enumerate(shapes)]
    xs = [bits_to_dev_bf16(synth.activations_bf16(21 + i, 1, K)) for i, (N, K) in enumerate(shapes)]
    nbytes = max(w4.workspace_bytes(1, N, K) for N, K in shapes)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    first = [None] * len(shapes)
    for rep in range(4):
        for i, (N, K) in enumerate(shapes):
            Y = torch.full((1, N), float("nan"), dtype=torch.bfloat16, device="cuda")
            w4.linear(xs[i], packs[i].qweight, packs[i].scales, packs[i].zeros, Y, ws, path=w4.PATH_DECODE)
            if first[i] is None:
                first[i] = Y
            else:
                torch.cuda.synchronize()
                assert torch.equal(Y.view(torch.int16), first[i].view(torch.int16)), (rep, N, K)
    torch.cuda.synchronize()
    assert not ws[:COUNTER_BYTES].any().item()
    N, K = shapes[0]
    X = synth.activations_bf16(21, 1, K)
    ref = _oracle_rows(N, K, 11, X, np.arange(N))
    assert_close(bf16_dev_to_f64(first[0]), ref, "interleaved 1000 x 2048")


@pytest.mark.parametrize("group", [64, 32])
def test_small_group_kernel_chunks_share_the_counter(cuda_lib, group):
    """The one-token kernel for groups of 64 and 32 deals its chunks from the same counter: repeated calls,
    interleaved with group-128 calls on one workspace, give the same bits and leave the counters at zero."""
    N, K = 3000, 4096
    W = dev_weights(41, synth.TAG_W, N, K)
    pw = w4.PackedWeight(N, K, group=group)
    pw.status = torch.zeros(1, dtype=torch.int32, device="cuda")
    w4.quantize_pack_g(W, group, pw.qweight, pw.scales, pw.zeros, pw.status)
    p128 = _packed(5120, 5120, 42)
    X = bits_to_dev_bf16(synth.activations_bf16(43, 1, K))
    X128 = bits_to_dev_bf16(synth.activations_bf16(44, 1, 5120))
    nbytes = max(w4.workspace_bytes_g(1, N, K, group), w4.workspace_bytes(1, 5120, 5120))
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(3):
        Y = torch.full((1, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        w4.linear_g(X, group, pw.qweight, pw.scales, pw.zeros, Y, ws)
        Y128 = torch.empty((1, 5120), dtype=torch.bfloat16, device="cuda")
        w4.linear(X128, p128.qweight, p128.scales, p128.zeros, Y128, ws)
        outs.append(Y)
    torch.cuda.synchronize()
    assert int(pw.status.item()) == 0
    assert not ws[:COUNTER_BYTES].any().item()
    for Y in outs[1:]:
        assert torch.equal(Y.view(torch.int16), outs[0].view(torch.int16))
    Wh = synth.weights_f32(41, synth.TAG_W, N, K)
    st, qw, sc, z = oracle.quantize_pack_g(Wh, group)
    assert st == oracle.OK
    assert_close(bf16_dev_to_f64(outs[0]), oracle.linear_g(synth.activations_bf16(43, 1, K), qw, sc, z), f"G={group}")
