"""Basis files and resumable calibration (the binding's save_basis / load_basis / Calibration).

The file layout follows the pages' basis file (JSSA README, section 2: ``{'M': {layer:
Tensor[H_kv, r, d]}}``, a latent layer ``[1, r, kv_lora_rank]``; ``--save_grams`` adds the second
moments). The CPU tests round-trip a file; the GPU test shows that a calibration stopped after
half of its samples, saved, loaded and resumed gives the same second moments and basis as one
that ran in one go.
"""

import numpy as np
import pytest
import torch


def test_basis_file_round_trip(tmp_path):
    import token_level_sparse_fp8_b200 as J
    g = torch.Generator().manual_seed(3)
    bases = {0: torch.randn(8, 32, 128, generator=g), 5: torch.randn(8, 32, 128, generator=g),
             7: torch.randn(1, 64, 512, generator=g)}  # a latent layer
    cals = {0: J.Calibration(8, 128, "cpu", torch.randn(8, 128, 128, generator=g, dtype=torch.float64),
                             torch.randn(8, 128, 128, generator=g, dtype=torch.float64), samples=4096)}
    eig = {0: torch.randn(8, 128, generator=g, dtype=torch.float64)}
    path = str(tmp_path / "basis.pt")
    J.save_basis(path, bases, cals, eig)
    raw = torch.load(path, weights_only=True)
    assert set(raw["M"]) == {0, 5, 7}
    assert raw["M"][0].shape == (8, 32, 128) and raw["M"][7].shape == (1, 64, 512)
    assert raw["M"][5].dtype == torch.float32
    assert raw["grams"][0]["samples"] == 4096
    back = J.load_basis(path)
    for layer, m in bases.items():
        assert torch.equal(back["M"][layer], m.float())
    c = back["grams"][0]
    assert c.samples == 4096
    assert torch.equal(c.gram_q, cals[0].gram_q) and torch.equal(c.gram_k, cals[0].gram_k)
    assert torch.equal(back["eigvals"][0], eig[0])
    # the runtime's rank must match the basis
    with pytest.raises(ValueError):
        J.load_basis(path, rank=16)
    with pytest.raises(ValueError):
        J.save_basis(str(tmp_path / "bad.pt"), {0: torch.zeros(8, 128)})


def test_basis_file_without_grams(tmp_path):
    import token_level_sparse_fp8_b200 as J
    path = str(tmp_path / "b.pt")
    J.save_basis(path, {2: torch.eye(4).repeat(2, 1, 1)[:, :2]})
    back = J.load_basis(path, rank=2)
    assert "grams" not in back and back["M"][2].shape == (2, 2, 4)
    with pytest.raises(ValueError):
        torch.save({"weights": 1}, path)
        J.load_basis(path)


@pytest.mark.gpu
def test_resumed_calibration_matches_one_shot(tmp_path):
    import token_level_sparse_fp8_b200 as J
    from oracle import jssa as O
    from synth import WORKLOADS, layer_factors, sample_calibration
    w = WORKLOADS["tiny"]
    f = layer_factors(w.seed, 0, w.h_kv, w.d)
    q, k = sample_calibration(f, 4096, w.group, w.seed)
    q, k = q.cuda(), k.cuda()
    one = J.calibrate(q, k, w.rank, batch=4096)
    # first half, saved with its moments; then loaded in place of the running state and resumed
    acc = J.Calibration(w.h_kv, w.d)
    acc.add(q[:2048], k[:2048])
    m_half, _ = acc.basis(w.rank)
    path = str(tmp_path / "half.pt")
    J.save_basis(path, {0: m_half}, {0: acc})
    del acc
    back = J.load_basis(path, device="cuda", rank=w.rank)
    acc2 = back["grams"][0]
    assert acc2.samples == 2048
    acc2.add(q[2048:], k[2048:])
    assert acc2.samples == 4096
    m2, e2 = acc2.basis(w.rank)
    torch.cuda.synchronize()
    for a, b in ((acc2.gram_q, one["gram_q"]), (acc2.gram_k, one["gram_k"])):
        a, b = a.cpu().numpy(), b.cpu().numpy()
        assert np.max(np.abs(a - b)) <= 1e-12 * np.max(np.abs(b))
    for h in range(w.h_kv):
        p1 = O.projector(m2[h].double().cpu().numpy())
        p0 = O.projector(one["M"][h].double().cpu().numpy())
        assert np.max(np.abs(p1 - p0)) <= 1e-6
    assert np.max(np.abs(e2.cpu().numpy() - one["eigvals"].cpu().numpy())) <= 1e-10
