"""The layer-step input recipe: seeded, shaped as documented, skewed per token block."""
import torch

import synthetic


def test_layer_step_inputs_shapes_seed_and_block_skew():
    w = synthetic.WORKLOADS["tiny"]
    a = synthetic.make_layer_step_inputs(w, 2, "cpu", seed=3)
    b = synthetic.make_layer_step_inputs(w, 2, "cpu", seed=3)
    T, hidden = w.total_tokens, w.hq * w.d
    assert a["x"].shape == (T, hidden) and a["g"].shape == (T, hidden)
    assert [t.shape for t in a["wqkv"]] == [(hidden, (w.hq + 2 * w.hkv) * w.d)] * 2
    assert [t.shape for t in a["wo"]] == [(hidden, hidden)] * 2
    assert all(torch.equal(a[k], b[k]) for k in ("x", "g"))
    # one scale per token block, shared by every head: per-block head norms stay in a fixed ratio
    g = a["g"].float().reshape(T // w.block, w.block, w.hq, w.d)
    per_block = g.norm(dim=(1, 3))                       # [blocks, heads]
    ratio = per_block / per_block.mean(dim=1, keepdim=True)
    assert float(ratio.std(dim=0).max()) < 0.5           # heads move together across blocks
    assert float(per_block.mean(dim=1).max() / per_block.mean(dim=1).min()) > 2.0   # blocks differ
