"""Data parallelism over tokens, world size 2 on CPU (gloo): each rank runs the
backward on its token shard, the flat parameter-gradient buffer is summed over
ranks, and the result must equal the backward over all tokens.  Also checks
the token sharding and the max-over-ranks reduction used for timing."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, result_dir, alpha, n):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    import torch.distributed as dist

    import oracle
    from manifold_constrained_hyper_token_b200 import parallel, synth
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    T, C = 37, 16
    d = synth.layer_inputs(T, n, C, seed=3, dtype=torch.float32, backward=True)
    lo, hi = parallel.token_shard(T, rank, world)
    r = oracle.backward(d["x"][lo:hi], d["phi"], d["b"], alpha, d["f_out"][lo:hi],
                        d["grad_x_next"][lo:hi], d["grad_h_in"][lo:hi], iters=20)
    flat, gphi, gb, ga = parallel.param_grad_buffer(n, C, "cpu", torch.float64,
                                                    alpha_groups=len(alpha))
    gphi.copy_(torch.from_numpy(r["grad_phi"]))
    gb.copy_(torch.from_numpy(r["grad_b"]))
    ga.copy_(torch.from_numpy(np.atleast_1d(np.asarray(r["grad_alpha"], dtype=np.float64))))
    parallel.allreduce_param_grads(flat)
    slowest = parallel.max_over_ranks(10.0 + rank, "cpu")
    np.save(os.path.join(result_dir, f"flat{rank}.npy"), flat.numpy())
    np.save(os.path.join(result_dir, f"gx{rank}.npy"), r["grad_x"])
    np.save(os.path.join(result_dir, f"max{rank}.npy"), np.array([slowest]))
    dist.barrier()
    dist.destroy_process_group()


def test_token_shard_covers_all_tokens():
    from manifold_constrained_hyper_token_b200 import parallel
    for T in (1, 7, 16384, 16385):
        for world in (1, 2, 3, 8):
            spans = [parallel.token_shard(T, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == T
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [e - s for s, e in spans]
            assert max(sizes) - min(sizes) <= 1


@pytest.mark.parametrize("n,alpha", [(4, [0.3]), (4, [0.3, -0.2, 0.5]), (8, [0.3, -0.2, 0.5]),
                                     (16, [0.3])],
                         ids=["n4_shared_alpha", "n4_alpha_groups3", "n8_alpha_groups3",
                              "n16_shared_alpha"])
def test_two_rank_backward_matches_single(tmp_path, n, alpha):
    import oracle
    from manifold_constrained_hyper_token_b200 import synth
    oracle.build()
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path), alpha, n),
                       nprocs=world, join=True, start_method="spawn")
    T, C = 37, 16
    d = synth.layer_inputs(T, n, C, seed=3, dtype=torch.float32, backward=True)
    full = oracle.backward(d["x"], d["phi"], d["b"], alpha, d["f_out"], d["grad_x_next"],
                           d["grad_h_in"], iters=20)
    K, M = n * C, n * n + 2 * n
    flats = [np.load(tmp_path / f"flat{r}.npy") for r in range(world)]
    np.testing.assert_array_equal(flats[0], flats[1])  # every rank holds the same sum
    np.testing.assert_allclose(flats[0][:K * M].reshape(K, M), full["grad_phi"], rtol=1e-12,
                               atol=1e-12)
    np.testing.assert_allclose(flats[0][K * M:K * M + M], full["grad_b"], rtol=1e-12, atol=1e-12)
    na = len(alpha)
    assert flats[0].size == K * M + M + na  # the buffer holds one grad_alpha per group
    np.testing.assert_allclose(flats[0][K * M + M:], np.atleast_1d(full["grad_alpha"]),
                               rtol=1e-12, atol=1e-12)
    gx = np.concatenate([np.load(tmp_path / f"gx{r}.npy") for r in range(world)])
    np.testing.assert_array_equal(gx, full["grad_x"])  # per-token outputs need no exchange
    assert all(np.load(tmp_path / f"max{r}.npy")[0] == 11.0 for r in range(world))
