"""Host logic of an RDR plan (compressed_kv_decode_ada_b200/rdr.py): physical
page allocation of the packed pages, on CPU tensors (no kernel runs)."""
import numpy as np
import pytest
import torch

import oracle


def _plan_from_oracle_pack(tier_lists, maxp=None):
    """A plan dict as spkv_rdr_plan returns it, with the pages of oracle.rdr_pack."""
    packs = [oracle.rdr_pack(np.asarray(t)) for t in tier_lists]
    B = len(packs)
    maxp = maxp or max([1] + [len(p[1]) for p in packs])
    bits = np.zeros((B, maxp), np.uint8)
    keep = np.zeros((B, maxp), np.uint16)
    for s, (_, pb, pk) in enumerate(packs):
        bits[s, :len(pb)] = pb
        keep[s, :len(pk)] = pk
    return {
        "tier": torch.from_numpy(np.concatenate([np.asarray(t, np.uint8) for t in tier_lists])),
        "dst_pos": torch.from_numpy(np.concatenate([p[0] for p in packs])),
        "page_bits": torch.from_numpy(bits),
        "page_keep": torch.from_numpy(keep.view(np.int16)),
        "n_pages": torch.tensor([len(p[1]) for p in packs], dtype=torch.int32),
        "status": torch.zeros(B, dtype=torch.int32),
    }, packs


def test_allocate_packed_lays_sequences_out_back_to_back():
    from compressed_kv_decode_ada_b200 import rdr

    rng = np.random.default_rng(0)
    tiers = [rng.choice([0, 3, 4, 6, 8], size=n) for n in (37, 0, 200, 16)]
    plan, packs = _plan_from_oracle_pack(tiers)
    cache, bt, ctx = rdr.allocate_packed(plan, 2, np.zeros(2, np.float32), np.ones(2, np.float32), device="cpu")
    n = [len(p[1]) for p in packs]
    assert cache.num_pages == sum(n)
    np.testing.assert_array_equal(ctx.numpy(), np.array(n) * 16)
    base = 0
    for s in range(len(tiers)):
        np.testing.assert_array_equal(bt[s, :n[s]].numpy(), base + np.arange(n[s]))
        np.testing.assert_array_equal(cache.page_bits[base:base + n[s]], packs[s][1])
        km = cache.keep_mask.numpy().view(np.uint16).reshape(-1, 2)
        for h in range(2):  # one decision per token: every kv head keeps the same slots
            np.testing.assert_array_equal(km[base:base + n[s], h], packs[s][2])
        base += n[s]


def test_allocate_packed_refuses_failed_plans():
    from compressed_kv_decode_ada_b200 import rdr

    plan, _ = _plan_from_oracle_pack([[3, 4, 8]])
    plan["status"] = torch.tensor([2], dtype=torch.int32)  # SPKV_RDR_PAGES
    with pytest.raises(ValueError):
        rdr.allocate_packed(plan, 1, np.zeros(1, np.float32), np.ones(1, np.float32), device="cpu")
    plan["status"] = torch.tensor([1], dtype=torch.int32)  # infeasible: still a valid plan
    cache, _, ctx = rdr.allocate_packed(plan, 1, np.zeros(1, np.float32), np.ones(1, np.float32), device="cpu")
    assert cache.num_pages == 3 and int(ctx[0]) == 48
