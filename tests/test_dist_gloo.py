"""The multi-process path on CPU: two gloo ranks (127.0.0.1) exercise the candidate sharding of sign selection (one
all-gather of per-candidate MSEs), the decode-unit sharding and the max-over-ranks timing reduction.  The scores
here come from a stand-in function of the candidates, since the CUDA path needs a GPU; what is tested is the
plumbing around it."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from kv_cache_quantized_b200 import dist as D


def _port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _fake_score(q, k, v, cands, bits, causal):
    # a deterministic stand-in objective: depends on the candidate's signs only
    w = torch.arange(1, cands.shape[1] + 1, dtype=torch.float64)
    return (cands.to(torch.float64) @ w) ** 2 / (1.0 + bits)


def _worker(rank, size, port, n_cand, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=size, init_method=f"tcp://127.0.0.1:{port}")
    try:
        rng = np.random.default_rng(0)
        cands = torch.from_numpy(np.where(rng.random((n_cand, 8)) < 0.5, -1, 1).astype(np.int8))
        mse, best = D.select_signs_sharded(None, None, None, cands, 3, score_fn=_fake_score)
        lo, hi = D.shard_range(16, rank, size)
        t = D.max_over_ranks([float(rank + 1), 10.0 - rank])
        np.save(os.path.join(out_dir, f"r{rank}.npy"),
                np.concatenate([mse.numpy(), [best, lo, hi, t[0], t[1]]]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("n_cand", [7, 200])
def test_sharded_selection_two_ranks(tmp_path, n_cand):
    size = 2
    mp.spawn(_worker, args=(size, _port(), n_cand, str(tmp_path)), nprocs=size, join=True)
    rng = np.random.default_rng(0)
    cands = torch.from_numpy(np.where(rng.random((n_cand, 8)) < 0.5, -1, 1).astype(np.int8))
    want = _fake_score(None, None, None, cands, 3, True).numpy()
    want_best = int(np.argmin(want))
    res = [np.load(tmp_path / f"r{r}.npy") for r in range(size)]
    for r, x in enumerate(res):
        assert np.array_equal(x[:n_cand], want)
        assert int(x[n_cand]) == want_best
        lo, hi = D.shard_range(16, r, size)
        assert (int(x[n_cand + 1]), int(x[n_cand + 2])) == (lo, hi)
        assert x[n_cand + 3] == 2.0 and x[n_cand + 4] == 10.0  # max over ranks
    # the shares tile the range exactly
    assert [D.shard_range(16, r, 2) for r in range(2)] == [(0, 8), (8, 16)]


def test_shard_range_covers_everything():
    for n in (0, 1, 7, 200, 201):
        for size in (1, 2, 3, 8):
            parts = [D.shard_range(n, r, size) for r in range(size)]
            assert parts[0][0] == 0 and parts[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(parts, parts[1:]))
            assert max(h - l for l, h in parts) - min(h - l for l, h in parts) <= 1


def test_single_process_identity():
    mse = torch.tensor([3.0, 1.0, 1.0, 2.0], dtype=torch.float64)
    assert D.first_argmin(mse) == 1
    assert torch.equal(D.gather_candidate_mse(mse, 4), mse)
    assert D.max_over_ranks([1.5]) == [1.5]


def _fake_score_layers(q, k, v, cands, bits, causal):
    # per layer a different deterministic stand-in objective of the candidate's signs
    w = torch.arange(1, cands.shape[1] + 1, dtype=torch.float64)
    base = (cands.to(torch.float64) @ w) ** 2
    return torch.stack([base / (1.0 + layer) + (layer * 7.0) % 5 * cands[:, layer % cands.shape[1]].double()
                        for layer in range(q.shape[0])])


def _worker_layers(rank, size, port, n_cand, out_dir):
    dist.init_process_group("gloo", rank=rank, world_size=size, init_method=f"tcp://127.0.0.1:{port}")
    try:
        rng = np.random.default_rng(1)
        cands = torch.from_numpy(np.where(rng.random((n_cand, 8)) < 0.5, -1, 1).astype(np.int8))
        q = torch.zeros((3, 1, 1, 1, 8))
        mse, best = D.select_signs_per_layer_sharded(q, None, None, cands, 2, score_fn=_fake_score_layers)
        np.save(os.path.join(out_dir, f"l{rank}.npy"), np.concatenate([mse.numpy().ravel(), best]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("n_cand", [5, 200])
def test_sharded_per_layer_selection_two_ranks(tmp_path, n_cand):
    size = 2
    mp.spawn(_worker_layers, args=(size, _port(), n_cand, str(tmp_path)), nprocs=size, join=True)
    rng = np.random.default_rng(1)
    cands = torch.from_numpy(np.where(rng.random((n_cand, 8)) < 0.5, -1, 1).astype(np.int8))
    want = _fake_score_layers(torch.zeros((3, 1, 1, 1, 8)), None, None, cands, 2, True).numpy()
    for r in range(size):
        x = np.load(tmp_path / f"l{r}.npy")
        assert np.array_equal(x[:3 * n_cand].reshape(3, n_cand), want)
        assert list(x[3 * n_cand:].astype(int)) == [int(np.argmin(want[layer])) for layer in range(3)]
