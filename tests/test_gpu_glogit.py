"""GPU parity of gla_fwd_glogit (bf16 gate logits, log_alpha = logsigmoid(g) / gate_norm
inside the tensor-core kernel) against the fp64 oracle (oracle.gla_fwd_glogit) on the
same bf16 logits, with the bf16 gates of tests/test_gpu_parity.py.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads

from test_gpu_parity import check_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dig():
    import gated_linear_attention_chunkwise_b200 as pkg
    return pkg


def run(dig, w, direction, seed=0, g=None, gate_norm=16.0, heads=None):
    q, k, v, g0 = workloads.gla_inputs_glogit(w, seed=seed)
    g = g0 if g is None else g
    out = dig.gla_fwd_glogit(q.cuda(), k.cuda(), v.cuda(), g.cuda(), w.Hgrid, w.Wgrid, direction, gate_norm=gate_norm)
    torch.cuda.synchronize()
    assert dig.device_status() == 0
    got = out.float().cpu().numpy().astype(np.float64)
    ref = oracle.gla_fwd_glogit(q, k, v, g, w.Hgrid, w.Wgrid, direction, gate_norm)
    check_bf16(got, ref, f"glogit dir {direction}", scan=(w.Hgrid, w.Wgrid, direction))


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_glogit_small(dig, direction):
    """A 9x23 grid (ragged chunks, column pieces) with d = 72."""
    run(dig, workloads.custom(2, 2, 9, 23, 72, 72, "bf16"), direction, seed=1)


@pytest.mark.parametrize("direction", [0, 3])
def test_glogit_c2(dig, direction):
    run(dig, workloads.WORKLOADS["c2"], direction, seed=2)


def test_glogit_c3_gate_mean_two_and_other_norm(dig):
    """DiG-B/2 at 1024 (g ~ N(2,1)), and gate_norm 4 on a small grid."""
    run(dig, workloads.WORKLOADS["c3"], 2, seed=3)
    run(dig, workloads.custom(1, 2, 16, 16, 64, 64, "bf16"), 1, seed=4, gate_norm=4.0)


def test_glogit_resets_and_open_gates(dig):
    """-inf logits (alpha = 0: full resets, token-serial chunks) and +inf (alpha = 1)."""
    w = workloads.custom(2, 2, 12, 17, 64, 64, "bf16")
    g = workloads.gla_inputs_glogit(w, seed=5)[3].float()
    m = torch.rand(g.shape, generator=torch.Generator().manual_seed(6))
    g = torch.where(m < 0.003, torch.full_like(g, -math.inf), g)
    g = torch.where(m > 0.99, torch.full_like(g, math.inf), g)
    for direction in (0, 2):
        run(dig, w, direction, seed=5, g=g.to(torch.bfloat16))


def test_glogit_rejects(dig):
    L = dig.lib()
    w = workloads.custom(1, 1, 4, 4, 128, 64, "bf16")
    q, k, v, g = (t.cuda() for t in workloads.gla_inputs_glogit(w))
    out = torch.empty_like(v)
    st = torch.cuda.current_stream().cuda_stream
    args = [q.data_ptr(), k.data_ptr(), v.data_ptr(), g.data_ptr(), 1, 1, 4, 4, 128, 64]
    assert L.gla_fwd_glogit(*args, 0, 16.0, out.data_ptr(), st) == -2    # dk > 120: the padded box
    args[8] = 64
    assert L.gla_fwd_glogit(*args, 4, 16.0, out.data_ptr(), st) == -2    # zigzag codes not here
    assert L.gla_fwd_glogit(*args, 0, 0.0, out.data_ptr(), st) == -1     # gate_norm must be positive
    assert dig.device_status() == 0
