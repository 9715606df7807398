"""Host logic of the sequence-parallel forward on CPU: which rows each shard
exchanges, checked against the brute-force key sets, and the whole exchange
run by gloo ranks with the oracle attending each rank's shard."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sparse_long_sequence_attn_b200 import seqpar
from sparse_long_sequence_attn_b200 import workloads as wl

# (N, H, patterns): aligned and partial last segments, a segment longer than
# the sequence, patterns local to a shard mixed with long ones.
CASES = [
    (64, 4, [(16, 1), (32, 2), (64, 4)]),
    (96, 3, [(8, 1), (48, 2), (96, 4)]),
    (80, 2, [(16, 1), (40, 2), (128, 8)]),
    (48, 5, [(6, 1), (24, 3), (36, 4)]),
]


def _brute_needed(B, N, H, patterns, G, g, causal):
    from oracle.brute import keys_reaching

    s0, s1 = seqpar.shard_bounds(N, G, g)
    need = set()
    for h in range(H):
        for pos in range(s0, s1):
            for kp in keys_reaching(pos, h, patterns, causal, N):
                if not (s0 <= kp < s1):
                    need.add(kp * H + h)
    one = np.array(sorted(need), dtype=np.int64)
    return np.concatenate([b * N * H + one for b in range(B)]) if len(one) else one


@pytest.mark.parametrize("N,H,patterns", CASES)
@pytest.mark.parametrize("G", [2, 4])
@pytest.mark.parametrize("causal", [True, False])
def test_needed_rows_match_brute_force_and_are_exchanged(N, H, patterns, G, causal):
    if N % G:
        pytest.skip("shards must be equal")
    B = 2
    lists = seqpar.exchange_lists(B, N, H, patterns, G)
    for g in range(G):
        need = seqpar.needed_rows(B, N, H, patterns, G, g, causal)
        assert np.array_equal(need, _brute_needed(B, N, H, patterns, G, g, causal))
        others = np.concatenate([lists[gg] for gg in range(G) if gg != g] + [np.zeros(0, np.int64)])
        assert np.isin(need, others).all(), "a needed row is exchanged by no other shard"
        s0, s1 = seqpar.shard_bounds(N, G, g)
        pos = (lists[g] // H) % N
        assert ((pos >= s0) & (pos < s1)).all() and np.all(np.diff(lists[g]) > 0)


def test_exchange_is_a_fraction_of_the_shard():
    # the dilation keeps about w / r of every w positions per head: with the
    # long pattern (N, 16) on 4 shards the exchanged rows are 1/16 of a shard
    B, N, H = 1, 1024, 16
    lists = seqpar.exchange_lists(B, N, H, [(64, 1), (N, 16)], 4)
    assert all(len(x) == (N // 4) * H // 16 for x in lists)


def test_local_patterns_exchange_nothing():
    B, N, H = 1, 256, 4
    assert seqpar.long_patterns([(32, 1), (64, 2), (128, 4)], N, 2) == []
    assert all(len(x) == 0 for x in seqpar.exchange_lists(B, N, H, [(32, 1), (128, 4)], 2))
    # a segment equal to the shard is local; one that does not tile the shard
    # (64 into 96 rows: the segment [64, 128) straddles the split) is long
    assert seqpar.long_patterns([(96, 2)], 192, 2) == []
    assert seqpar.long_patterns([(64, 2)], 192, 2) == [(64, 2)]


def test_shard_bounds_rejects_uneven_split():
    with pytest.raises(ValueError):
        seqpar.shard_bounds(100, 3, 0)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _gather(src, idx, dst):
    dst.copy_(src.reshape(-1, src.shape[-1])[idx])


def _scatter(src, idx, dst):
    dst.view(-1, dst.shape[-1])[idx] = src


def _rank_main(rank, world, port, outdir, N, H, patterns, causal):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle

        w = wl.WORKLOADS["tiny"]
        q, k, v = (x.double() for x in wl.make_inputs(w, N=N, H=H))
        B, D = q.shape[0], q.shape[-1]
        s0, s1 = seqpar.shard_bounds(N, world, rank)
        # what this rank holds: its own shard; everything else NaN until exchanged
        kf = torch.full_like(k, float("nan"))
        vf = torch.full_like(v, float("nan"))
        qf = torch.full_like(q, float("nan"))
        kf[:, s0:s1], vf[:, s0:s1], qf[:, s0:s1] = k[:, s0:s1], v[:, s0:s1], q[:, s0:s1]
        sent = seqpar.exchange_kv(kf, vf, patterns, gather=_gather, scatter=_scatter)
        rows = np.array([(b, x, h) for b in range(B) for x in range(s0, s1) for h in range(H)], np.int64)
        out, lse = oracle.dilated_attn_rows_fp64(qf.numpy(), kf.numpy(), vf.numpy(), patterns, rows, causal)
        np.save(os.path.join(outdir, f"out{rank}.npy"), out.reshape(B, s1 - s0, H, D))
        np.save(os.path.join(outdir, f"lse{rank}.npy"), lse.reshape(B, s1 - s0, H))
        np.save(os.path.join(outdir, f"sent{rank}.npy"), np.array([sent]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("causal", [True, False])
def test_gloo_ranks_exchange_then_attend_their_shard(tmp_path, world, causal):
    """Every rank holds only its shard (NaN elsewhere), exchanges the kept rows
    of the long patterns over gloo, and the oracle attends for the rank's rows
    on what it then holds: the result is bit-identical to the single-process
    oracle, so every row the shard reads arrived and nothing else is read."""
    N, H = 128, 4
    patterns = [(16, 1), (64, 2), (128, 4)]
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path), N, H, patterns, causal),
             nprocs=world, join=True)
    import oracle

    w = wl.WORKLOADS["tiny"]
    q, k, v = (x.double().numpy() for x in wl.make_inputs(w, N=N, H=H))
    ref, ref_lse = oracle.dilated_attn_fp64(q, k, v, patterns, causal)
    got = np.concatenate([np.load(tmp_path / f"out{r}.npy") for r in range(world)], axis=1)
    got_lse = np.concatenate([np.load(tmp_path / f"lse{r}.npy") for r in range(world)], axis=1)
    assert np.array_equal(got, ref)
    assert np.array_equal(got_lse.transpose(0, 2, 1), ref_lse)
    sent = [int(np.load(tmp_path / f"sent{r}.npy")[0]) for r in range(world)]
    assert all(s > 0 for s in sent)
