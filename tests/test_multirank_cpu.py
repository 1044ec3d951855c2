"""The multi-rank path on CPU: two gloo ranks shard the requests, all-gather the
survival scores, run the same scheduler on the global batch and keep their slices.

The scheduler here is the CPU oracle (a GPU is not needed to check the exchange and
the slicing that bench.py uses with NCCL).
"""
import os
import socket

import numpy as np
import pytest

import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, B, gamma, out_dir):
    import torch
    import torch.distributed as dist

    import oracle
    from speculative_decoding_drafter_head_b200 import sharding

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        P_all = synth.monotone_scores(B * world, gamma, seed=11, tie_frac=0.25)
        b0 = sharding.request_offset(rank, B)
        P_local = torch.from_numpy(P_all[b0:b0 + B].copy())
        P_glob = sharding.gather_scores(P_local)
        wl = synth.Workload("multirank", B=B * world, gamma=gamma, V=100, sps_knee=B * world + 8)
        L, N, F, _ = oracle.schedule(P_glob.numpy(), synth.tstep_us(wl))
        L_loc = sharding.local_lengths(torch.from_numpy(L), rank, B).numpy()
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), P=P_glob.numpy(), L=L, N=N, F=F,
                 L_loc=L_loc)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_two_ranks_agree_on_global_schedule(tmp_path, oracle_mod, world):
    import torch.multiprocessing as mp
    B, gamma = 7, 5
    mp.spawn(_worker, args=(world, _free_port(), B, gamma, str(tmp_path)), nprocs=world,
             join=True)
    P_all = synth.monotone_scores(B * world, gamma, seed=11, tie_frac=0.25)
    wl = synth.Workload("multirank", B=B * world, gamma=gamma, V=100, sps_knee=B * world + 8)
    L_ref, N_ref, F_ref, _ = oracle_mod.schedule(P_all, synth.tstep_us(wl))
    assert 0 < N_ref < B * world * gamma          # the knee makes some drafts not worth verifying
    parts = []
    for r in range(world):
        d = np.load(tmp_path / f"rank{r}.npz")
        np.testing.assert_array_equal(d["P"], P_all)
        np.testing.assert_array_equal(d["L"], L_ref)
        assert int(d["N"]) == N_ref and float(d["F"]) == F_ref
        parts.append(d["L_loc"])
    np.testing.assert_array_equal(np.concatenate(parts), L_ref)


def test_noise_keys_use_global_request_index(oracle_mod):
    """A shard drafted with its global request ids equals the same rows of the full batch."""
    V, r, gamma, B = 300, 8, 4, 6
    rng = np.random.default_rng(2)
    U = synth.f32_to_bf16_bits(rng.normal(0, 1, (B, gamma, V)).astype(np.float32))
    W1 = synth.f32_to_bf16_bits(rng.normal(0, 0.3, (V, r)).astype(np.float32))
    W2 = synth.f32_to_bf16_bits(rng.normal(0, 0.3, (r, V)).astype(np.float32))
    anchor = rng.integers(0, V, B).astype(np.int32)
    full, _, _ = oracle_mod.draft(U, anchor, W1, W2, mode=1, tau=0.8, seed=5)
    shard, _, _ = oracle_mod.draft(U[3:], anchor[3:], W1, W2, mode=1, tau=0.8, seed=5,
                                   b_index=np.arange(3, B, dtype=np.int32))
    np.testing.assert_array_equal(shard, full[3:])


def test_rnn_noise_keys_use_global_request_index(oracle_mod):
    """The RNN head drafted on a shard with its global request ids equals the same rows of
    the full batch (the state is per request, so sharding by request keeps it local)."""
    V, r, gamma, B = 300, 8, 4, 6
    rng = np.random.default_rng(3)
    U = synth.f32_to_bf16_bits(rng.normal(0, 1, (B, gamma, V)).astype(np.float32))
    W1 = synth.f32_to_bf16_bits(rng.normal(0, 0.3, (V, r)).astype(np.float32))
    W2 = synth.f32_to_bf16_bits(rng.normal(0, 0.3, (r, V)).astype(np.float32))
    Whh = synth.f32_to_bf16_bits(rng.normal(0, 0.2, (r, r)).astype(np.float32))
    anchor = rng.integers(0, V, B).astype(np.int32)
    full, _, _ = oracle_mod.draft_rnn(U, anchor, W1, W2, Whh, mode=1, tau=0.8, seed=5)
    shard, _, _ = oracle_mod.draft_rnn(U[2:], anchor[2:], W1, W2, Whh, mode=1, tau=0.8, seed=5,
                                       b_index=np.arange(2, B, dtype=np.int32))
    np.testing.assert_array_equal(shard, full[2:])
