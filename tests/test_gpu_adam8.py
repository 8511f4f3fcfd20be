"""GPU parity of the AdamW step with 8-bit blockwise state (qlora_adamw8_step)
against the oracle through the C-ABI: parameters, both moments' codes and
absmax values bit-exact after every one of several steps, on adapter-shaped
tensors with a partial final block, and the bf16 copy of the parameters."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import nf4_oracle as o

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import bit_nf4_quantised_b200 as pkg
    pkg.lib()
    return pkg


f32 = lambda x: float(np.float32(x))


@pytest.mark.parametrize("shape", [(16, 4096), (4096, 16), (24, 768), (3, 100), (1, 1)])
def test_adamw8_matches_oracle(q, shape):
    rng = np.random.default_rng(shape[0] * 7 + shape[1])
    n = shape[0] * shape[1]
    p = (rng.standard_normal(n) * 0.02).astype(np.float32)
    hp = dict(lr=f32(2e-4), beta1=f32(0.9), beta2=f32(0.999), eps=f32(1e-8),
              weight_decay=f32(0.01))
    pd = torch.from_numpy(p.copy()).cuda()
    st = q.adamw8_state(n)
    pb = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    ms = o.encode_state8(np.zeros(n, np.float32), True, 64)
    vs = o.encode_state8(np.zeros(n, np.float32), False, 64)
    for t in range(1, 6):
        g = rng.standard_normal(n).astype(np.float32)
        if t == 3:
            g[:64] = 0.0                        # a block whose gradient vanishes
        q.qlora_adamw8_step(pd, torch.from_numpy(g).cuda(), st, p_bf16=pb, **hp)
        p, ms, vs = o.adamw8_step(p, g, ms, vs, t, hp["lr"], hp["beta1"], hp["beta2"],
                                  hp["eps"], hp["weight_decay"])
        torch.cuda.synchronize()
        assert np.array_equal(pd.cpu().numpy().view(np.uint32), p.view(np.uint32)), t
        assert np.array_equal(st.m_codes.cpu().numpy(), ms[0]), t
        assert np.array_equal(st.m_absmax.cpu().numpy().view(np.uint32), ms[1].view(np.uint32)), t
        assert np.array_equal(st.v_codes.cpu().numpy(), vs[0]), t
        assert np.array_equal(st.v_absmax.cpu().numpy().view(np.uint32), vs[1].view(np.uint32)), t
        assert np.array_equal(pb.view(torch.int16).cpu().numpy().view(np.uint16), o.bf16_bits(p)), t


def test_adamw8_wide_dynamic_range(q):
    """Gradients whose blocks span 1e-30 .. 1e30 (and signed zeros), so that
    the moments, their bias-corrected values and their block quotients fall
    both inside and outside the range where the kernel divides by a
    reciprocal and two fused multiply-adds; every result must still carry the
    correctly rounded bits the oracle's fp32 divisions give."""
    rng = np.random.default_rng(77)
    n = 64 * 96
    p = (rng.standard_normal(n) * 0.02).astype(np.float32)
    hp = dict(lr=f32(1e-3), beta1=f32(0.9), beta2=f32(0.999), eps=f32(1e-8),
              weight_decay=f32(0.0))
    pd = torch.from_numpy(p.copy()).cuda()
    st = q.adamw8_state(n)
    ms = o.encode_state8(np.zeros(n, np.float32), True, 64)
    vs = o.encode_state8(np.zeros(n, np.float32), False, 64)
    scale = np.repeat(10.0 ** rng.uniform(-30, 18, n // 64), 64).astype(np.float32)
    for t in range(1, 5):
        g = (rng.standard_normal(n).astype(np.float32) * scale).astype(np.float32)
        g[64:72] = np.float32(-0.0)                 # signed zeros inside a live block
        g[128:192] *= np.float32(1e-12)             # a block far below its neighbours
        q.qlora_adamw8_step(pd, torch.from_numpy(g).cuda(), st, **hp)
        p, ms, vs = o.adamw8_step(p, g, ms, vs, t, hp["lr"], hp["beta1"], hp["beta2"],
                                  hp["eps"], hp["weight_decay"])
        torch.cuda.synchronize()
        assert np.array_equal(pd.cpu().numpy().view(np.uint32), p.view(np.uint32)), t
        assert np.array_equal(st.m_codes.cpu().numpy(), ms[0]), t
        assert np.array_equal(st.m_absmax.cpu().numpy().view(np.uint32), ms[1].view(np.uint32)), t
        assert np.array_equal(st.v_codes.cpu().numpy(), vs[0]), t
        assert np.array_equal(st.v_absmax.cpu().numpy().view(np.uint32), vs[1].view(np.uint32)), t
