"""GPU parity of the router training loss L_aux (forward and backward) against the CPU oracle.

Tolerance: the kernel computes in fp32 from bf16 inputs; the oracle in fp64 on the same
inputs.  The loss agrees to 1e-5 relative.  A gradient element is a difference of two
products (the cosine's direction term minus its norm term), so its fp32 error is bounded
by the size of those terms, not of the result: each element must lie within
1e-4 * max|oracle| + 1e-3 * |oracle| of the oracle's value.
"""
import numpy as np
import pytest

import oracle as O
from long_context_memory_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msa(cuda_device):
    import long_context_memory_b200 as m

    return m


def _close(gpu, ref, what):
    scale = np.max(np.abs(ref)) if ref.size else 0.0
    bound = 1e-4 * scale + 1e-3 * np.abs(ref)
    err = np.abs(gpu - ref)
    assert np.all(err <= bound), f"{what}: worst excess {np.max(err - bound):.3e} (scale {scale:.3e})"


def _case(seed, P, N, n_r, d_r, pos_scale=0.6):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((P, n_r, d_r))
    Kp = Q + pos_scale * rng.standard_normal((P, n_r, d_r))       # positives lean toward the query
    Kn = rng.standard_normal((P, N, n_r, d_r))
    b = lambda a: W.f32_to_bf16_bits(a.astype(np.float32))
    return b(Q), b(Kp), b(Kn)


# (the last two: more negatives than stay resident in shared memory, so the rows stream twice;
# at d_r = 128 with 1023 negatives the ring is cut to what shared memory holds)
@pytest.mark.parametrize("P,N,n_r,d_r,tau", [(1, 0, 8, 128, 0.1), (5, 7, 8, 128, 0.05), (33, 63, 4, 64, 0.2),
                                             (300, 15, 3, 128, 1.0), (2, 1023, 8, 64, 0.07),
                                             (3, 1023, 8, 128, 0.07)])
def test_aux_loss_parity(msa, cuda_device, P, N, n_r, d_r, tau):
    import torch

    Q, Kp, Kn = _case(P * 7 + N, P, N, n_r, d_r)
    dims = W.Dims(hidden=256, n_q=8, n_kv=2, head_dim=64, n_r=n_r, d_r=d_r)
    dev = cuda_device
    t = lambda a: W.to_torch(np.ascontiguousarray(a)).to(dev)
    loss, dQ, dKp, dKn = msa.aux_loss(dims, t(Q), t(Kp), t(Kn) if N else None, tau)
    torch.cuda.synchronize()
    assert msa.check_device_errors() == 0
    l_o, dQ_o, dKp_o, dKn_o = O.aux_loss(Q, Kp, Kn, tau)
    assert abs(loss.item() - l_o) <= 1e-5 * max(1.0, abs(l_o)), (loss.item(), l_o)
    _close(dQ.cpu().numpy(), dQ_o, "dQR")
    _close(dKp.cpu().numpy(), dKp_o, "dK_pos")
    if N:
        _close(dKn.cpu().numpy(), dKn_o, "dK_neg")


def test_aux_loss_zero_vectors_and_loss_only(msa, cuda_device):
    # a zero query head and a zero key head: cosine 0, no gradient through the clamped norm
    import torch

    Q, Kp, Kn = _case(5, 4, 6, 2, 64)
    Q[1, 0] = 0
    Kn[2, 3, 1] = 0
    dims = W.Dims(hidden=256, n_q=8, n_kv=2, head_dim=64, n_r=2, d_r=64)
    t = lambda a: W.to_torch(np.ascontiguousarray(a)).to(cuda_device)
    loss, dQ, dKp, dKn = msa.aux_loss(dims, t(Q), t(Kp), t(Kn), 0.1)
    loss_only = msa.aux_loss(dims, t(Q), t(Kp), t(Kn), 0.1, grads=False)[0]
    torch.cuda.synchronize()
    l_o, dQ_o, dKp_o, dKn_o = O.aux_loss(Q, Kp, Kn, 0.1)
    assert abs(loss.item() - l_o) <= 1e-5 * max(1.0, abs(l_o))
    assert loss_only.item() == loss.item()
    _close(dQ.cpu().numpy(), dQ_o, "dQR")
    _close(dKn.cpu().numpy(), dKn_o, "dK_neg")


def test_aux_loss_deterministic(msa, cuda_device):
    import torch

    Q, Kp, Kn = _case(9, 1000, 31, 8, 128)
    dims = W.QWEN3_4B_DIMS
    t = lambda a: W.to_torch(np.ascontiguousarray(a)).to(cuda_device)
    a = msa.aux_loss(dims, t(Q), t(Kp), t(Kn), 0.05)
    b = msa.aux_loss(dims, t(Q), t(Kp), t(Kn), 0.05)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)
