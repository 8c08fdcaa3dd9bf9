"""GPU parity for the sequence split across ranks: every rank's local steps
(la_state_local, la_state_range_sum, la_forward_sp, la_backward_sp_dq,
la_backward_sp_dkdv) through the C ABI, with the shards' outputs put back
together and compared with the fp64 oracle's forward and backward over the
whole sequence.  States are sums over tokens ("Efficient Transformers
Survey", Proposition "Linear Attention via Kernel Decomposition",
Statement), so the sharded results must equal the unsharded ones.

Ranks are emulated one after another on one GPU (the all-gather becomes a
stack of the records: nothing waits across ranks), and, through
seqpar.forward / backward, as two processes on the one GPU exchanging
records over gloo (host collectives; the kernels of the two processes never
wait on each other)."""
import datetime
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from linear_attention_transformers_b200 import api, inputs, seqpar
from parity_util import compare, relu_branch_as_kernel

pytestmark = pytest.mark.gpu

PHIS = {"elu1": oracle.PHI_ELU1, "relu_eps": oracle.PHI_RELU_EPS}


def sharded(q, k, v, dO, lens, causal, phi):
    """All ranks' steps, rank by rank; returns the concatenated o, dq, dk, dv
    and the kernels launched."""
    P = len(lens)
    cuts = np.cumsum([0] + list(lens))
    sh = [[t[:, :, cuts[r]:cuts[r + 1]].contiguous() for t in (q, k, v, dO)] for r in range(P)]
    api.la_profile_enable(True)
    api.la_profile_collect()
    # forward: local records -> (all-gather) -> prefix sums -> local pass
    recs = torch.stack([api.la_state_local(s[1], s[2], phi) for s in sh])
    outs = []
    for r, (qr, kr, vr, _) in enumerate(sh):
        state_in = api.la_state_range_sum(recs, *seqpar.prefix_range(r, P, causal))
        g = torch.empty(qr.shape[:3], dtype=torch.float32, device=q.device)
        outs.append((api.la_forward_sp(qr, kr, vr, state_in, causal, phi, g=g), g))
    # backward: centred records -> dQ step -> query-side records -> dK/dV step
    crecs = torch.stack([api.la_state_local(s[1], s[2], phi, centred=True) for s in sh])
    dqs, rrecs, wss = [], [], []
    for r, (qr, kr, vr, dOr) in enumerate(sh):
        state_in = api.la_state_range_sum(crecs, *seqpar.prefix_range(r, P, causal))
        o, g = outs[r]
        dq, rrec, ws = api.la_backward_sp_dq(qr, kr, vr, dOr, o, g, state_in, causal, phi)
        dqs.append(dq)
        rrecs.append(rrec)
        wss.append(ws)
    rrecs = torch.stack(rrecs)
    dks, dvs = [], []
    for r, (qr, kr, vr, dOr) in enumerate(sh):
        r_in = api.la_state_range_sum(rrecs, *seqpar.suffix_range(r, P, causal))
        dk, dv = api.la_backward_sp_dkdv(qr, kr, vr, dOr, outs[r][1], r_in, wss[r], causal, phi)
        dks.append(dk)
        dvs.append(dv)
    torch.cuda.synchronize()
    api.la_get_device_error()
    ran = set(api.la_profile_collect())
    api.la_profile_enable(False)
    cat = lambda xs: torch.cat(xs, dim=2)  # noqa: E731
    return cat([o for o, _ in outs]), cat(dqs), cat(dks), cat(dvs), ran


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("phi", ["elu1", "relu_eps"])
@pytest.mark.parametrize("lens", [(300, 129, 0, 348), (1000, 129, 600)])
def test_sharded_matches_whole_sequence(D, causal, phi, lens):
    N = sum(lens)
    q, k, v, dO = (t.cuda() for t in inputs.make_tensors(2, 3, N, D, torch.bfloat16,
                                                         seed=N + D, with_grad_out=True))
    o, dq, dk, dv, ran = sharded(q, k, v, dO, lens, causal, phi)
    assert {"state_range_sum", "bwd_dq", "bwd_dkdv"} <= ran, ran
    assert ("reduce128" if D == 128 else "chunk_reduce") in ran, ran
    assert ("chunk_causal" if causal else "chunk_query") in ran, ran
    o_ref, _, _ = oracle.forward(q, k, v, causal, PHIS[phi])
    rq, rk, rv = oracle.backward(q, k, v, dO, causal, PHIS[phi])
    if phi == "relu_eps":
        rq, rk = relu_branch_as_kernel(rq, q), relu_branch_as_kernel(rk, k)
    compare(o, o_ref, torch.bfloat16, "o")
    compare(dq, rq, torch.bfloat16, "dq")
    compare(dk, rk, torch.bfloat16, "dk")
    compare(dv, rv, torch.bfloat16, "dv")


def test_sharded_many_heads_one_segment_each():
    # 128 heads: every shard runs one block per head (no segment split)
    lens = (256, 384)
    q, k, v, dO = (t.cuda() for t in inputs.make_tensors(4, 32, sum(lens), 64, torch.bfloat16,
                                                         seed=77, with_grad_out=True))
    o, dq, dk, dv, _ = sharded(q, k, v, dO, lens, True, "elu1")
    o_ref, _, _ = oracle.forward(q, k, v, True, oracle.PHI_ELU1)
    rq, rk, rv = oracle.backward(q, k, v, dO, True, oracle.PHI_ELU1)
    compare(o, o_ref, torch.bfloat16, "o")
    compare(dq, rq, torch.bfloat16, "dq")
    compare(dk, rk, torch.bfloat16, "dk")
    compare(dv, rv, torch.bfloat16, "dv")


def test_state_chain_equals_whole_sequence_state():
    # the causal forward's state_out of shard r is shard r+1's state_in, and
    # the last one is la_forward's final state of the whole sequence
    lens = (200, 333)
    q, k, v = (t.cuda() for t in inputs.make_tensors(1, 4, sum(lens), 128, torch.bfloat16,
                                                     seed=9))
    B, H, N, D = q.shape
    state = torch.zeros((B, H, D * D + D), dtype=torch.float32, device="cuda")
    a = 0
    for n in lens:
        nxt = torch.empty_like(state)
        api.la_forward_sp(*(t[:, :, a:a + n].contiguous() for t in (q, k, v)), state, True,
                          "elu1", state_out=nxt)
        state, a = nxt, a + n
    _, S, z = api.la_forward(q, k, v, True, "elu1", return_state=True)
    torch.cuda.synchronize()
    want = torch.cat([S.reshape(B, H, D * D), z], dim=2)
    scale = want.abs().max().item()
    assert (state - want).abs().max().item() <= 4e-3 * scale


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, lens, outdir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v, dO = inputs.make_tensors(2, 4, sum(lens), 64, torch.bfloat16, seed=21,
                                          with_grad_out=True)
        a = sum(lens[:rank])
        qr, kr, vr, dOr = (t[:, :, a:a + lens[rank]].contiguous().cuda() for t in (q, k, v, dO))
        o, g = seqpar.forward(qr, kr, vr, True, "elu1")
        dq, dk, dv = seqpar.backward(qr, kr, vr, dOr, o, g, True, "elu1")
        torch.cuda.synchronize()
        api.la_get_device_error()
        torch.save({n: t.cpu() for n, t in (("o", o), ("dq", dq), ("dk", dk), ("dv", dv))},
                   os.path.join(outdir, f"r{rank}.pt"))
    finally:
        dist.destroy_process_group()


def test_two_processes_over_gloo():
    lens = (513, 700)
    with tempfile.TemporaryDirectory() as d:
        mp.spawn(_rank_main, args=(2, _free_port(), lens, d), nprocs=2, join=True)
        res = [torch.load(os.path.join(d, f"r{r}.pt")) for r in range(2)]
    q, k, v, dO = inputs.make_tensors(2, 4, sum(lens), 64, torch.bfloat16, seed=21,
                                      with_grad_out=True)
    o_ref, _, _ = oracle.forward(q, k, v, True, oracle.PHI_ELU1)
    rq, rk, rv = oracle.backward(q, k, v, dO, True, oracle.PHI_ELU1)
    for name, ref in (("o", o_ref), ("dq", rq), ("dk", rk), ("dv", rv)):
        compare(torch.cat([res[0][name], res[1][name]], dim=2), ref, torch.bfloat16, name)


def _rank_autograd(rank, world, port, lens, outdir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v, dO = inputs.make_tensors(1, 4, sum(lens), 128, torch.bfloat16, seed=23,
                                          with_grad_out=True)
        a = sum(lens[:rank])
        qr, kr, vr = (t[:, :, a:a + lens[rank]].contiguous().cuda().requires_grad_(True)
                      for t in (q, k, v))
        dOr = dO[:, :, a:a + lens[rank]].contiguous().cuda()
        o = seqpar.SequenceParallelLinearAttention.apply(qr, kr, vr, True, "relu_eps")
        o.backward(dOr)
        torch.cuda.synchronize()
        api.la_get_device_error()
        torch.save({n: t.detach().cpu() for n, t in (("o", o), ("dq", qr.grad), ("dk", kr.grad),
                                                    ("dv", vr.grad))},
                   os.path.join(outdir, f"r{rank}.pt"))
    finally:
        dist.destroy_process_group()


def test_autograd_wrapper_two_processes():
    # torch autograd over the split sequence (head size 128, relu+eps)
    lens = (700, 300)
    with tempfile.TemporaryDirectory() as d:
        mp.spawn(_rank_autograd, args=(2, _free_port(), lens, d), nprocs=2, join=True)
        res = [torch.load(os.path.join(d, f"r{r}.pt")) for r in range(2)]
    q, k, v, dO = inputs.make_tensors(1, 4, sum(lens), 128, torch.bfloat16, seed=23,
                                      with_grad_out=True)
    o_ref, _, _ = oracle.forward(q, k, v, True, oracle.PHI_RELU_EPS)
    rq, rk, rv = oracle.backward(q, k, v, dO, True, oracle.PHI_RELU_EPS)
    rq, rk = relu_branch_as_kernel(rq, q), relu_branch_as_kernel(rk, k)
    for name, ref in (("o", o_ref), ("dq", rq), ("dk", rk), ("dv", rv)):
        compare(torch.cat([res[0][name], res[1][name]], dim=2), ref, torch.bfloat16, name)


@pytest.mark.parametrize("lens", [(1, 1, 1), (128, 1, 127, 0, 256), (64, 64), (5, 500, 3)])
@pytest.mark.parametrize("D", [64, 128])
def test_sharded_edge_lengths(lens, D):
    # one-token shards, shards on and off chunk boundaries, empty shards,
    # five ranks, a single head
    N = sum(lens)
    q, k, v, dO = (t.cuda() for t in inputs.make_tensors(1, 1, N, D, torch.bfloat16,
                                                         seed=3 * N + D, with_grad_out=True))
    for causal in (True, False):
        o, dq, dk, dv, _ = sharded(q, k, v, dO, lens, causal, "elu1")
        o_ref, _, _ = oracle.forward(q, k, v, causal, oracle.PHI_ELU1)
        rq, rk, rv = oracle.backward(q, k, v, dO, causal, oracle.PHI_ELU1)
        compare(o, o_ref, torch.bfloat16, "o")
        compare(dq, rq, torch.bfloat16, "dq")
        compare(dk, rk, torch.bfloat16, "dk")
        compare(dv, rv, torch.bfloat16, "dv")
