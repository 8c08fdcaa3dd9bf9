"""Host-side checks of the sequence split across ranks
(linear_attention_transformers_b200.seqpar): which ranks' records each rank
sums, that the all-gather hands them over in rank order (gloo, world sizes
2 and 3, on CPU), and that the C entry points refuse bad arguments before
they launch anything.  The records here are the fp64 oracle's final states
of each shard, so the exchanged prefix must equal the oracle's state of the
whole prefix (states are sums over tokens: "Efficient Transformers Survey",
Proposition "Linear Attention via Kernel Decomposition", Statement)."""
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from linear_attention_transformers_b200 import api, build, inputs, seqpar


def test_ranges():
    assert seqpar.prefix_range(0, 4, True) == (0, 0)
    assert seqpar.prefix_range(2, 4, True) == (0, 2)
    assert seqpar.prefix_range(2, 4, False) == (0, 4)
    assert seqpar.suffix_range(3, 4, True) == (4, 4)
    assert seqpar.suffix_range(1, 4, True) == (2, 4)
    assert seqpar.suffix_range(1, 4, False) == (0, 4)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _record(S, z):
    """[B, H, D, D] and [B, H, D] -> [B, H, D*D + D] records."""
    B, H, D, _ = S.shape
    return torch.from_numpy(np.concatenate([S.reshape(B, H, D * D), z], axis=2))


def _rank_main(rank, world, port, shards, outdir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        q, k, v = shards[rank]
        _, S, z = oracle.forward(q, k, v, True, oracle.PHI_ELU1)
        rec = _record(S, z)
        def combine(g, lo, hi):
            return g[lo:hi].sum(0)
        pre = seqpar.exchange(rec, seqpar.prefix_range(rank, world, True), combine=combine)
        tot = seqpar.exchange(rec, seqpar.prefix_range(rank, world, False), combine=combine)
        suf = seqpar.exchange(rec, seqpar.suffix_range(rank, world, True), combine=combine)
        torch.save({"pre": pre, "tot": tot, "suf": suf}, os.path.join(outdir, f"r{rank}.pt"))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_exchange_over_gloo_gives_prefix_total_and_suffix_states(world):
    B, H, D = 1, 2, 8
    lens = [5, 7, 3][:world]
    q, k, v = (t.double().numpy() for t in inputs.make_tensors(B, H, sum(lens), D,
                                                                  torch.float32, 5))
    cuts = np.cumsum([0] + lens)
    shards = [tuple(np.ascontiguousarray(t[:, :, cuts[r]:cuts[r + 1]]) for t in (q, k, v))
              for r in range(world)]
    with tempfile.TemporaryDirectory() as d:
        mp.spawn(_rank_main, args=(world, _free_port(), shards, d), nprocs=world, join=True)
        res = [torch.load(os.path.join(d, f"r{r}.pt")) for r in range(world)]
    for r in range(world):
        # the oracle's own state of tokens [0, cuts[r]) (prefix), of all, and
        # of tokens after shard r
        _, S, z = oracle.forward(q[:, :, :max(cuts[r], 1)], k[:, :, :max(cuts[r], 1)],
                                 v[:, :, :max(cuts[r], 1)], True, oracle.PHI_ELU1)
        want_pre = _record(S, z).numpy() if cuts[r] > 0 else np.zeros((B, H, D * D + D))
        _, S, z = oracle.forward(q, k, v, True, oracle.PHI_ELU1)
        want_tot = _record(S, z).numpy()
        np.testing.assert_allclose(res[r]["pre"].numpy(), want_pre, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(res[r]["tot"].numpy(), want_tot, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(res[r]["suf"].numpy(), want_tot - want_pre -
                                   _record(*oracle.forward(*shards[r], True,
                                                           oracle.PHI_ELU1)[1:]).numpy(),
                                   rtol=1e-10, atol=1e-12)


FAKE = 0x100000  # aligned, non-null, never dereferenced


@pytest.fixture(scope="module")
def lib():
    build.build()
    return api.load_library()


def test_sp_calls_reject_bad_arguments_before_launch(lib):
    B, H, N, D = 1, 2, 100, 64
    bf, f32 = api.LA_BF16, api.LA_F32
    # range sum: 0 <= lo <= hi <= P
    assert lib.la_state_range_sum(FAKE, 2, 1, 0, FAKE, B, H, D, None) == api.LA_ERR_INVALID_ARG
    assert lib.la_state_range_sum(FAKE, 2, 0, 3, FAKE, B, H, D, None) == api.LA_ERR_INVALID_ARG
    assert lib.la_state_range_sum(FAKE, 2, 0, 1, None, B, H, D, None) == api.LA_ERR_INVALID_ARG
    assert lib.la_state_range_sum(FAKE, 2, 0, 1, FAKE, B, H, 48, None) == api.LA_ERR_UNSUPPORTED
    # tensor-core path only: float32 and head sizes 16, 32 are refused
    assert lib.la_state_local(FAKE, FAKE, FAKE, B, H, N, D, f32, 0, 0, None, 0,
                              None) == api.LA_ERR_UNSUPPORTED
    assert lib.la_state_local(FAKE, FAKE, FAKE, B, H, N, 32, bf, 0, 0, None, 0,
                              None) == api.LA_ERR_UNSUPPORTED
    assert lib.la_state_local(FAKE, FAKE, None, B, H, N, D, bf, 0, 0, None, 0,
                              None) == api.LA_ERR_INVALID_ARG
    # forward: state_in required, state_out causal only, workspace checked
    assert lib.la_forward_sp(FAKE, FAKE, FAKE, FAKE, None, None, None, B, H, N, D, bf, 1, 0,
                             None, 0, None) == api.LA_ERR_INVALID_ARG
    assert lib.la_forward_sp(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, B, H, N, D, bf, 0, 0,
                             None, 0, None) == api.LA_ERR_INVALID_ARG
    need_b = lib.la_workspace_size_sp(api.LA_OP_BACKWARD, B, H, N, D, 1, bf)
    assert need_b >= B * H * N * 4  # dg at least
    assert lib.la_backward_sp_dq(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, B, H, N,
                                 D, bf, 1, 0, None, 0, None) == api.LA_ERR_WORKSPACE
    assert lib.la_backward_sp_dq(FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, B, H, N,
                                 D, bf, 1, 0, FAKE, need_b, None) == api.LA_ERR_INVALID_ARG
    assert lib.la_backward_sp_dkdv(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, B, H, N, D,
                                   bf, 1, 0, FAKE, need_b - 256, None) == api.LA_ERR_WORKSPACE
    assert lib.la_backward_sp_dkdv(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, B, H, N, D,
                                   bf, 1, 0, FAKE, need_b, None) == api.LA_ERR_INVALID_ARG
    assert lib.la_workspace_size_sp(api.LA_OP_FORWARD, B, H, N, D, 1, f32) == 0
