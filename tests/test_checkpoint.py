"""Basis files and resumable calibration (the binding's save_basis / load_basis / Calibration).

The file layout follows the pages' basis file (JSSA README, section 2: ``{'M': {layer:
Tensor[H_kv, r, d]}}``, a latent layer ``[1, r, kv_lora_rank]``; ``--save_grams`` adds the second
moments). The CPU tests round-trip a file; the GPU test shows that a calibration stopped after
half of its samples, saved, loaded and resumed gives the same second moments and basis as one
that ran in one go. A data-parallel calibration sums its ranks' moments with
``Calibration.all_reduce``: two gloo ranks on CPU, each with its own samples, end with identical
moments equal to the oracle's over all samples, and the same basis; on the GPU the same call
runs through an NCCL group of one rank.
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


def _reduce_rank(rank, world, port, out):
    # one rank of a data-parallel calibration: the moments of this rank's own samples, summed
    # over the ranks by Calibration.all_reduce on a gloo group
    import os
    import sys
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    import torch.distributed as dist
    import token_level_sparse_fp8_b200 as J
    from oracle import jssa as O
    from synth import layer_factors, sample_calibration
    dist.init_process_group("gloo", rank=rank, world_size=world)
    f = layer_factors(1700, 0, 2, 64)
    q, k = sample_calibration(f, 300, 4, 1700 + rank)  # this rank's samples
    g_q, g_k = O.second_moments(O.group_mean_query(q.double().numpy(), 2), k.double().numpy())
    cal = J.Calibration(2, 64, "cpu", torch.from_numpy(g_q), torch.from_numpy(g_k), samples=300)
    cal.all_reduce()
    dist.destroy_process_group()
    out.put((rank, cal.gram_q.numpy(), cal.gram_k.numpy(), cal.samples))


def test_calibration_all_reduce_two_gloo_ranks():
    import multiprocessing as mp
    import socket
    from oracle import jssa as O
    from synth import layer_factors, sample_calibration
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_reduce_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((out.get(timeout=120) for _ in procs), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (_, q0, k0, n0), (_, q1, k1, n1) = res
    # every rank holds the same moments: those of both ranks' samples together
    assert np.array_equal(q0, q1) and np.array_equal(k0, k1) and n0 == n1 == 600
    f = layer_factors(1700, 0, 2, 64)
    qs, ks = zip(*(sample_calibration(f, 300, 4, 1700 + r) for r in range(2)))
    q, k = torch.cat(qs).double().numpy(), torch.cat(ks).double().numpy()
    g_q, g_k = O.second_moments(O.group_mean_query(q, 2), k)
    np.testing.assert_allclose(q0, g_q, rtol=1e-12, atol=1e-9)
    np.testing.assert_allclose(k0, g_k, rtol=1e-12, atol=1e-9)
    # and the basis solved from the reduced moments is the one-shot calibration's
    m_red, _ = O.joint_basis(q0, k0, 16)
    m_one, _ = O.joint_basis(g_q, g_k, 16)
    p_red = np.einsum("hri,hrj->hij", m_red, m_red)
    p_one = np.einsum("hri,hrj->hij", m_one, m_one)
    np.testing.assert_allclose(p_red, p_one, atol=1e-9)


def _nccl_single_rank(port, out):
    # Calibration.all_reduce on the GPU's own moments through an NCCL group of one rank
    import os
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import torch.distributed as dist
    import token_level_sparse_fp8_b200 as J
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    g = torch.Generator(device="cuda").manual_seed(5)
    gq = torch.randn(8, 128, 128, generator=g, dtype=torch.float64, device="cuda")
    gk = torch.randn(8, 128, 128, generator=g, dtype=torch.float64, device="cuda")
    cal = J.Calibration(8, 128, "cuda", gq.clone(), gk.clone(), samples=1234)
    cal.all_reduce()
    ok = (torch.equal(cal.gram_q, gq) and torch.equal(cal.gram_k, gk) and cal.samples == 1234
          and cal.gram_q.is_cuda)
    dist.destroy_process_group()
    out.put(ok)


@pytest.mark.gpu
def test_calibration_all_reduce_nccl_single_rank():
    import multiprocessing as mp
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    p = ctx.Process(target=_nccl_single_rank, args=(port, out))
    p.start()
    ok = out.get(timeout=300)
    p.join(timeout=60)
    assert p.exitcode == 0 and ok
