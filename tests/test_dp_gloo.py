"""Data-parallel path on CPU: world_size-2 gloo process groups.

The host logic of the multi-GPU step is the sharding of the global batch over
ranks and one all-reduce (sum) of the flat LoRA gradient buffer.  Here two
ranks each run the oracle's sparse FFN forward/backward on their own shard
(with their own contextual selection) and sum their gradients through
dp.allreduce_grads; the result must equal the sum of the per-shard oracle
gradients computed in one process.  A rank that never joins makes the others
fail within the bounded timeout instead of hanging."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from oracle import slora_oracle as O
from contextual_sparsity_lora_svd_b200 import dp, synth

GRAD_KEYS = ("dAg", "dBg", "dAu", "dBu", "dAd", "dBd")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _global_case():
    tok = synth.Tokens(4, 24, np.asarray([18, 24, 9, 16], np.int32))
    case = synth.ffn_case(tok, 32, 80, 4, 3, 0.5, bf16=False, workload=0, layer=9)
    lay = dict(Wg=case.Wg.W, Wu=case.Wu.W, Wd=case.Wd.W, Ag=case.Ag, Bg=case.Bg, Au=case.Au,
               Bu=case.Bu, Ad=case.Ad, Bd=case.Bd, scale=case.lora_scale)
    lay["Lg"], lay["Ug"] = O.svd_prepare(case.Wg.W, 4)
    lay["Lu"], lay["Uu"] = O.svd_prepare(case.Wu.W, 4)
    return tok, case, lay


def _shard_grads(tok, case, lay, start, count):
    """Oracle gradients of sequences [start, start + count) with their own selection."""
    rows = slice(start * tok.seq, (start + count) * tok.seq)
    X, dOut = case.X[rows], case.dOut[rows]
    ctx = tok.ctx_len[start:start + count]
    ref = O.ffn_fwd_bwd(X, dOut, count, tok.seq, ctx, lay, case.sparsity)
    return np.concatenate([np.asarray(ref[k], np.float64).ravel() for k in GRAD_KEYS]), ref["idx"]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    r, w = dp.init_from_env("gloo", timeout_s=60)
    tok, case, lay = _global_case()
    start, count = dp.shard(tok.batch, w, r)
    flat, idx = _shard_grads(tok, case, lay, start, count)
    t = torch.from_numpy(flat.copy())
    dp.allreduce_grads(t)
    worst = dp.max_over_ranks(float(r + 1))
    np.save(os.path.join(out_dir, f"rank{r}.npy"), t.numpy())
    np.save(os.path.join(out_dir, f"idx{r}.npy"), idx)
    np.save(os.path.join(out_dir, f"max{r}.npy"), np.asarray([worst]))
    torch.distributed.destroy_process_group()


def test_shard_partitions_the_batch():
    for batch in range(0, 19):
        for world in range(1, 9):
            blocks = [dp.shard(batch, world, r) for r in range(world)]
            covered = []
            for s, c in blocks:
                covered.extend(range(s, s + c))
            assert covered == list(range(batch)), (batch, world)
            sizes = [c for _, c in blocks]
            assert max(sizes) - min(sizes) <= 1
            assert sizes == sorted(sizes, reverse=True)
    with pytest.raises(ValueError):
        dp.shard(4, 2, 2)


def test_allreduce_is_noop_without_group():
    t = torch.arange(5, dtype=torch.float32)
    dp.allreduce_grads(t)
    assert torch.equal(t, torch.arange(5, dtype=torch.float32))
    assert dp.max_over_ranks(3.5) == 3.5


def test_two_rank_gradient_sum(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    tok, case, lay = _global_case()
    want = sum(_shard_grads(tok, case, lay, *dp.shard(tok.batch, world, r))[0]
               for r in range(world))
    for r in range(world):
        got = np.load(tmp_path / f"rank{r}.npy")
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-12 * np.abs(want).max())
        assert np.load(tmp_path / f"max{r}.npy")[0] == world
    # each rank selected from its own context tokens: the sets differ here
    i0, i1 = np.load(tmp_path / "idx0.npy"), np.load(tmp_path / "idx1.npy")
    assert i0.shape == i1.shape and not np.array_equal(i0, i1)
    # and the DP sum is not the single-batch gradient (selection is per shard)
    full, _ = _shard_grads(tok, case, lay, 0, tok.batch)
    assert np.abs(full - want).max() > 1e-9


def _lonely_rank(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    try:
        dp.init_from_env("gloo", timeout_s=3)
        outcome = "joined"
    except Exception as e:  # the peer never arrives
        outcome = type(e).__name__
    with open(os.path.join(out_dir, "outcome.txt"), "w") as f:
        f.write(outcome)


def test_missing_peer_times_out(tmp_path):
    """Rank 0 of a world of 2 whose rank 1 never starts: the rendezvous ends
    with an error within the bounded timeout."""
    port = _free_port()
    ctx = mp.get_context("spawn")
    p = ctx.Process(target=_lonely_rank, args=(0, 2, port, str(tmp_path)))
    p.start()
    p.join(timeout=120)
    if p.is_alive():
        p.kill()
        pytest.fail("rank 0 kept waiting for its missing peer")
    assert (tmp_path / "outcome.txt").read_text() != "joined"
