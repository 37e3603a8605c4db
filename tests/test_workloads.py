"""The seeded synthetic workloads hold the recipe they state (CPU, small sizes):
shapes, the log-normal per-channel scales (and the tiny law's outlier channels), a
block table that is a permutation, slot mappings that hit every slot once, one
generator chunk per prefill80 layer, sub-range reproducibility of the bulk
generator, and the query law."""
import math

import numpy as np
import pytest

from kv_cache_vector_02_b200 import workloads as W


def test_sizes_of_the_named_workloads():
    b = W.WORKLOADS["batched"]
    assert (b.B, b.T, b.Hkv, b.Hq) == (32, 4096, 8, 32) and b.tokens == 32 * 4096
    assert b.num_blocks == 32 * 256 and b.max_blocks == 256
    l70 = W.WORKLOADS["long70b"]
    assert (l70.B, l70.T, l70.Hkv, l70.Hq) == (1, 131072, 8, 64)
    p80 = W.WORKLOADS["prefill80"]
    assert p80.tokens == 80 * 32768 and p80.num_blocks == 80 * 32768 // 16
    l8 = W.WORKLOADS["llama8b"]
    assert l8.max_seq_len == 4096 + 64 and l8.max_blocks == (4096 + 64) // 16


@pytest.mark.parametrize("law,sig,n_out", [("llama8b", 0.5, 3), ("long70b", 0.7, 1)])
def test_channel_scales_follow_the_log_normal_law(law, sig, n_out):
    w = W.WORKLOADS[law]
    for kind in (0, 1):
        s = W.channel_scales(w, kind)
        assert s.shape == (w.Hkv, 128) and s.dtype == np.float32 and np.all(s > 0)
        # without each row's n_out largest (where the outlier channels sit), log s is
        # N(0, sig^2) up to sampling error and the trimming of its upper tail
        body = np.log(np.sort(s, axis=1)[:, : 128 - n_out]).ravel()
        assert abs(np.median(body)) < 0.15 and 0.8 * sig < body.std() < 1.1 * sig
    # the same call gives the same scales; K and V and layers differ
    assert np.array_equal(W.channel_scales(w, 0), W.channel_scales(w, 0))
    assert not np.array_equal(W.channel_scales(w, 0), W.channel_scales(w, 1))
    assert not np.array_equal(W.channel_scales(w, 0, 0), W.channel_scales(w, 0, 1))


def test_tiny_law_outlier_channels():
    w = W.WORKLOADS["tiny"]
    s = W.channel_scales(w, 0)
    assert np.array_equal(np.flatnonzero(s[0] == 10.0), [0, 32, 64, 96]) and np.all(np.delete(s[0], [0, 32, 64, 96]) == 1)
    assert np.all(W.channel_scales(w, 1) == 1)


def test_block_table_is_a_permutation_and_slots_are_unique():
    w = W.WORKLOADS["batched"].with_(B=5, T=100)
    bt = W.block_table(w)
    assert bt.shape == (5, w.max_blocks) and bt.dtype == np.int32
    assert np.array_equal(np.sort(bt.ravel()), np.arange(w.num_blocks))
    sl = W.prefill_slots(w, bt)
    assert sl.shape == (5 * 100,) and np.unique(sl).size == sl.size
    assert sl.min() >= 0 and sl.max() < w.num_blocks * 16
    # token t of sequence b sits in row t % 16 of block bt[b, t // 16]
    assert sl[3 * 100 + 37] == bt[3, 2] * 16 + 5
    w2 = w.with_(decode_steps=20)
    bt2 = W.block_table(w2)
    allsl = np.concatenate([W.prefill_slots(w2, bt2)] + [W.step_slots(w2, bt2, s) for s in range(20)])
    assert np.unique(allsl).size == allsl.size


def test_flat_slots_cover_the_pages():
    n = 16 * 7 + 5
    plain, perm = W.flat_slots(n), W.flat_slots(n, perm_seed=3)
    assert np.array_equal(plain, np.arange(n))
    assert np.unique(perm).size == n and np.array_equal(perm % 16, np.arange(n) % 16)
    assert np.array_equal(np.sort(np.unique(perm // 16)), np.arange(8))


def test_bulk_generator_subranges_and_laws():
    w = W.WORKLOADS["llama8b"].with_(T=40000)      # two generator chunks of 32768 tokens
    full = W.gen_kv(w, 1)
    assert full.shape == (40000, 8, 128) and str(full.dtype) == "torch.float16"
    part = W.gen_kv(w, 1, token_offset=32000, n_tokens=2000)   # straddles the chunk edge
    assert np.array_equal(part.numpy(), full[32000:34000].numpy())
    # per-channel std follows the scales within sampling error
    x = full.float().numpy()
    std = x.std(axis=0)
    s = W.channel_scales(w, 1)
    assert np.all(np.abs(std / s - 1) < 0.05)
    q = W.gen_q(W.WORKLOADS["batched"]).float().numpy()
    assert q.shape == (32, 32, 128) and abs(q.std() * math.sqrt(128) - 1) < 0.03


def test_prefill80_layers_draw_their_own_scales():
    """One generator chunk per layer (32768 tokens): layer 2's tokens follow layer 2's
    channel scales, not layer 0's."""
    w = W.WORKLOADS["prefill80"]
    x = W.gen_kv(w, 0, token_offset=2 * 32768, n_tokens=4096).float().numpy()
    std = x.std(axis=0)
    r2 = std / W.channel_scales(w, 0, 2)
    r0 = std / W.channel_scales(w, 0, 0)
    assert np.all(np.abs(r2 - 1) < 0.1)
    assert np.abs(r0 - 1).max() > 1.0
