"""The seeded input generator: deterministic, thread-count independent, and
drawing the distributions the workloads name."""

import numpy as np
import torch

import workloads as wl


def test_deterministic_and_thread_independent(monkeypatch):
    a = wl.normal_bf16(3, wl.TID_WGATE, (3000, 3000), std=0.02)
    monkeypatch.setattr(wl, "_threads", lambda: 1)
    b = wl.normal_bf16(3, wl.TID_WGATE, (3000, 3000), std=0.02)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    c = wl.normal_bf16(4, wl.TID_WGATE, (3000, 3000), std=0.02)
    assert not torch.equal(a.view(torch.int16), c.view(torch.int16))


def test_distributions():
    p = wl.make_problem(64, 1024, 688, sigma=0.02, seed=0, residual=True)
    assert p["x"].shape == (64, 1024) and p["x"].dtype == torch.bfloat16
    assert p["W_gate"].shape == (688, 1024) and p["W_down"].shape == (1024, 688)
    x = p["x"].double()
    assert abs(x.mean().item()) < 0.02 and abs(x.std().item() - 1) < 0.02
    g = p["gamma"].double()
    assert abs(g.mean().item() - 1) < 0.02 and abs(g.std().item() - 0.1) < 0.01
    for k in ("W_gate", "W_up", "W_down"):
        w = p[k].double()
        assert abs(w.std().item() - 0.02) < 5e-4
    # independent streams per tensor
    assert not torch.equal(p["W_gate"], p["W_up"])
    assert not torch.equal(p["x"], p["residual"])


def test_workload_table():
    w = wl.WORKLOADS
    assert (w["tiny"].M, w["tiny"].d, w["tiny"].I) == (4, 256, 688)
    assert (w["phi3_decode"].d, w["phi3_decode"].I, w["phi3_decode"].layers) == (3072, 8192, 32)
    assert w["llama70b_verify"].M == 128 and w["llama70b_verify"].sigma == 0.01
    assert w["llama8b_prefill"].M == 2048
    assert w["phi3_decode"].weight_bytes == 6 * 3072 * 8192


def test_bits_view_is_exact():
    t = wl.normal_bf16(0, 0, (5, 7))
    b = wl.bf16_bits(t)
    assert b.dtype == np.uint16 and b.shape == (5, 7)
    back = torch.from_numpy(b.view(np.int16)).view(torch.bfloat16)
    assert torch.equal(back.view(torch.int16), t.view(torch.int16))
