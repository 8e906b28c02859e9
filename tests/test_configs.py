"""Host-side checks of the workload table and the synthetic block state (CPU)."""
import torch

from block_diffusion_moe_dllm_b200 import configs, synth


def test_every_workload_splits_into_its_guidance_groups():
    for w in configs.ALL:
        assert w.cfg in (0, 1, 2), w.name
        assert w.B % (1 + w.cfg) == 0, w.name
        assert w.L <= 32 or (w.P == 0 and w.T_s == 1), w.name   # else the prefill shape: one block-causal pass
        assert w.cap == w.P + w.L, w.name
        assert 0 <= w.vocab_offset and w.vocab_offset + w.vlen <= w.V, w.name


def test_editing_guidance_runs_without_sprint():
    """Under editing guidance SPRINT falls back to the plain decode on the full caches (HF-mirror README, note under
    "SPRINT 加速技术"): a workload asking for both keeps the guidance and drops the retention."""
    w = configs.scaled(configs.EDIT, sprint=1, keep_ratio=0.5)
    assert w.cfg == 2 and w.sprint == 0 and w.n_keep == w.P
    assert configs.scaled(configs.T2I, sprint=1).sprint == 1   # two-way guidance keeps SPRINT


def test_block_state_shares_its_pattern_across_guidance_groups():
    for base, groups in ((configs.T2I, 2), (configs.EDIT, 3)):
        w = configs.scaled(base, B=2 * groups, V=1000, vocab_offset=0, vocab_len=0)
        tokens, mask = synth.make_block_state(w, "cpu", seed=5, masked_fraction=0.5)
        Bl = w.B // groups
        assert 0 < int(mask[:Bl].sum()) < Bl * w.L
        for g in range(1, groups):
            assert torch.equal(mask[g * Bl:(g + 1) * Bl], mask[:Bl])
            assert torch.equal(tokens[g * Bl:(g + 1) * Bl], tokens[:Bl])
        assert torch.all(tokens[mask.bool()] == w.mask_id)
