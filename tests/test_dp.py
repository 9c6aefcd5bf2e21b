"""Data parallelism over tokens (rank_linear_lora_b200.dp), on CPU with gloo ranks.

The per-rank gradients here come from the oracle (the CUDA path needs a GPU); what is
under test is the host logic the GPU path uses: the token split, the packed [dA | dB]
layout the backward writes into, and the one sum all-reduce.  The sum over ranks must
equal the gradient of the whole batch (dA and dB are sums over tokens)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import oracle
from rank_linear_lora_b200 import inputs
from rank_linear_lora_b200.dp import PackedGrads, token_shard


def test_token_shard_covers_every_row_once():
    for M in (0, 1, 2, 7, 64, 4097):
        for world in (1, 2, 3, 8):
            rows = []
            sizes = []
            for rank in range(world):
                start, count = token_shard(M, world, rank)
                rows.extend(range(start, start + count))
                sizes.append(count)
            assert rows == list(range(M))
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        token_shard(8, 2, 2)


def test_packed_views_are_the_kernel_layouts():
    g = PackedGrads(3, 5, 7)
    assert g.buf.numel() == 3 * 5 + 7 * 3 and g.buf.dtype == torch.float32
    assert g.dA.shape == (3, 5) and g.dA.is_contiguous() and g.dA.data_ptr() == g.buf.data_ptr()
    assert g.dB.shape == (7, 3) and g.dB.is_contiguous()
    assert g.dB.data_ptr() == g.buf.data_ptr() + 4 * 3 * 5
    g.dA.fill_(1.0)
    g.dB.fill_(2.0)
    assert g.buf[:15].eq(1.0).all() and g.buf[15:].eq(2.0).all()


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, spec, result_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = inputs.make_inputs(spec)  # the same global batch on every rank
        start, count = token_shard(spec.M, world, rank)
        grads = PackedGrads(spec.r, spec.d_in, spec.d_out)
        if count == 0:
            grads.zero_()
        else:
            x, dY = inp.x[start:start + count], inp.dY[start:start + count]
            bwd = oracle.backward(dY, x, inp.A, inp.B, spec.s, W=inp.W)
            # the backward writes fp32 into the packed views
            grads.dA.copy_(torch.from_numpy(bwd["dA"]).float())
            grads.dB.copy_(torch.from_numpy(bwd["dB"]).float())
        grads.all_reduce()
        np.save(os.path.join(result_dir, f"rank{rank}.npy"), grads.buf.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("M", [67, 1], ids=["ragged", "one-rank-empty"])
def test_allreduce_of_shards_equals_full_batch(tmp_path, M):
    world = 2
    spec = inputs.LayerSpec("dp", M, 256, 192, 8, alpha=16.0, seed=0xD9)
    mp.spawn(_worker, args=(world, _free_port(), spec, str(tmp_path)), nprocs=world, join=True)
    inp = inputs.make_inputs(spec)
    full = oracle.backward(inp.dY, inp.x, inp.A, inp.B, spec.s, W=inp.W)
    ref = np.concatenate([full["dA"].ravel(), full["dB"].ravel()])
    for rank in range(world):
        got = np.load(tmp_path / f"rank{rank}.npy").astype(np.float64)
        # each rank's part is rounded once to fp32 before the sum: error <= 2 ulp of fp32
        np.testing.assert_allclose(got, ref, rtol=0, atol=4e-7 * np.abs(ref).max())
    # every rank holds the same sum
    assert np.array_equal(np.load(tmp_path / "rank0.npy"), np.load(tmp_path / "rank1.npy"))


def _stack(M, d_in, d_outs, r, alpha, seed):
    """Projections of one x (per-projection seeded inputs) and their stacked layout."""
    from lora_cases import shared_input_projections
    from rank_linear_lora_b200.multi import SharedInputProjections

    layers = shared_input_projections(M, d_in, d_outs, r, alpha, False, seed)
    st = SharedInputProjections(d_in, d_outs, r, alpha)
    t16 = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)  # noqa: E731
    for p, inp in enumerate(layers):
        st.load(p, W=t16(inp.W), A=t16(inp.A), B=t16(inp.B))
    bits = lambda t: t.view(torch.int16).numpy().view(np.uint16)  # noqa: E731
    return layers, st, bits(st.W), bits(st.A), bits(st.B)


def _stack_worker(rank, world, port, case, result_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        M, d_in, d_outs, r, alpha, seed = case
        layers, st, W, A, B = _stack(*case)
        dY = np.concatenate([inp.dY for inp in layers], axis=1)
        start, count = token_shard(M, world, rank)
        bwd = oracle.backward(dY[start:start + count], layers[0].x[start:start + count], A, B,
                              st.alpha_call / st.r_call, W=W)
        st.grads.dA.copy_(torch.from_numpy(bwd["dA"]).float())
        st.grads.dB.copy_(torch.from_numpy(bwd["dB"]).float())
        st.grads.all_reduce()  # one collective for every projection of the stack
        np.save(os.path.join(result_dir, f"rank{rank}.npy"), st.grads.buf.numpy())
    finally:
        dist.destroy_process_group()


def test_stacked_projections_reduce_in_one_allreduce(tmp_path):
    """Projections of one x stacked into one layer: each rank's backward of its token
    shard fills the stack's packed buffer, one all-reduce sums it, and every
    projection's dA, dB view then holds that projection's whole-batch gradient."""
    world, case = 2, (41, 64, (24, 16), 8, 16.0, 0xDA)
    mp.spawn(_stack_worker, args=(world, _free_port(), case, str(tmp_path)), nprocs=world, join=True)
    layers, st, *_ = _stack(*case)
    for rank in range(world):
        st.grads.buf.copy_(torch.from_numpy(np.load(tmp_path / f"rank{rank}.npy")))
        for p, (dA_p, dB_p) in enumerate(st.split_grads()):
            inp = layers[p]
            full = oracle.backward(inp.dY, inp.x, inp.A, inp.B, inp.spec.s, W=inp.W)
            for got, ref in ((dA_p, full["dA"]), (dB_p, full["dB"])):
                np.testing.assert_allclose(got.numpy().astype(np.float64), ref, rtol=0,
                                           atol=4e-7 * np.abs(ref).max())
