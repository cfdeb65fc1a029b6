"""Guard regions and bit-exact repeats for the entry points beyond the forward:
the backward (four outputs), the normalised variant, the gate-logit forward and the
zigzag orders.  Each output lives inside a NaN-filled buffer with 4096 elements on
each side; the guards must stay NaN and a second call must agree bit for bit.
"""

import pytest
import torch

import workloads

from test_gpu_parity import _bits, _guarded, _guards_intact

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dig():
    import gated_linear_attention_chunkwise_b200 as pkg
    return pkg


def test_bwd_guarded_and_repeatable(dig):
    w = workloads.custom(2, 3, 10, 13, 72, 40, "bf16")
    q, k, v, la = (t.cuda() for t in workloads.gla_inputs(w, seed=21))
    do = workloads.gla_dout(w, seed=21).cuda()
    L = dig.lib()
    st = torch.cuda.current_stream().cuda_stream
    for d in (0, 2, 5):
        g = [_guarded((w.B, w.T, w.H, n), dt) for n, dt in ((w.dk, torch.bfloat16), (w.dk, torch.bfloat16),
                                                            (w.dv, torch.bfloat16), (w.dk, torch.float32))]
        rc = L.gla_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), la.data_ptr(), do.data_ptr(), w.B, w.H, w.Hgrid,
                       w.Wgrid, w.dk, w.dv, d, *[x[1].data_ptr() for x in g], st)
        assert rc == 0
        again = dig.gla_bwd(q, k, v, la, do, w.Hgrid, w.Wgrid, d)
        torch.cuda.synchronize()
        for (buf, out, guard, n), b in zip(g, again):
            assert torch.equal(_bits(out), _bits(b))
            assert _guards_intact(buf, guard, n)
    assert dig.device_status() == 0


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_norm_guarded_and_repeatable(dig, dtype):
    w = workloads.custom(2, 2, 9, 14, 64, 48, "bf16" if dtype == torch.bfloat16 else "f32")
    q, k, v, _ = (t.cuda() for t in workloads.gla_inputs(w, seed=22))
    fn = dig.gla_norm_fwd if dtype == torch.bfloat16 else dig.gla_norm_fwd_f32
    for d in (1, 3, 8):
        buf, out, guard, n = _guarded((w.B, w.T, w.H, w.dv), dtype)
        a = fn(q, k, v, w.Hgrid, w.Wgrid, d, out=out).clone()
        b = fn(q, k, v, w.Hgrid, w.Wgrid, d)
        assert torch.equal(_bits(a), _bits(b))
        assert _guards_intact(buf, guard, n)
    assert dig.device_status() == 0


def test_glogit_guarded_and_repeatable(dig):
    w = workloads.custom(2, 3, 10, 13, 72, 72, "bf16")
    q, k, v, g = (t.cuda() for t in workloads.gla_inputs_glogit(w, seed=23))
    for d in range(4):
        buf, out, guard, n = _guarded((w.B, w.T, w.H, w.dv), torch.bfloat16)
        a = dig.gla_fwd_glogit(q, k, v, g, w.Hgrid, w.Wgrid, d, out=out).clone()
        b = dig.gla_fwd_glogit(q, k, v, g, w.Hgrid, w.Wgrid, d)
        assert torch.equal(_bits(a), _bits(b))
        assert _guards_intact(buf, guard, n)
    assert dig.device_status() == 0


def test_zigzag_forward_guarded_and_repeatable(dig):
    w = workloads.custom(2, 3, 10, 13, 72, 72, "bf16")
    q, k, v, la = (t.cuda() for t in workloads.gla_inputs(w, seed=24))
    for j in (0, 5):
        buf, out, guard, n = _guarded((w.B, w.T, w.H, w.dv), torch.bfloat16)
        a = dig.gla_fwd(q, k, v, la, w.Hgrid, w.Wgrid, 4 + j, out=out).clone()
        b = dig.gla_fwd(q, k, v, la, w.Hgrid, w.Wgrid, 4 + j)
        assert torch.equal(_bits(a), _bits(b))
        assert _guards_intact(buf, guard, n)
    assert dig.device_status() == 0
