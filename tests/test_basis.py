"""The rotated-basis set-up (no GPU): orthonormal directions, dot products
preserved, directions ordered by their share of score variance."""
import dataclasses

import torch

from long_context_decode_bit_b200 import basis, inputs


def test_klt_basis_properties():
    w = dataclasses.replace(inputs.STEP_1M_LLAMA, H=3, n=6000, seed=9)
    k = inputs.keys(w, 0, w.H)
    q = inputs.queries(w, 0, w.H).float()
    U = basis.klt_basis(k[:, :4096], q)
    eye = torch.eye(w.D).expand(w.H, -1, -1)
    assert torch.allclose(U.transpose(1, 2) @ U, eye, atol=1e-5)
    kr, qr = basis.rotate(k, U), basis.rotate(q, U)
    ref = q.double() @ k.double().transpose(1, 2)
    rot = qr.double() @ kr.double().transpose(1, 2)
    assert torch.allclose(rot, ref, rtol=0, atol=1e-4 * float(ref.abs().max()))
    # the trace of the key covariance is preserved
    x = k[:, :4096].double()
    xr = kr[:, :4096].double()
    assert torch.allclose(x.var(1, unbiased=False).sum(1), xr.var(1, unbiased=False).sum(1), rtol=1e-5)
    # ordering: lambda_i * u_i^T Sigma_q u_i is non-increasing along the columns
    cov = torch.einsum("hnd,hne->hde", x - x.mean(1, keepdim=True), x - x.mean(1, keepdim=True)) / 4096
    lam = torch.einsum("hdi,hde,hei->hi", U.double(), cov, U.double())
    sq = q.double().transpose(1, 2) @ q.double()
    wgt = lam * torch.einsum("hdi,hde,hei->hi", U.double(), sq, U.double())
    assert torch.all(wgt[:, :-1] >= wgt[:, 1:] - 1e-9 * wgt.abs().max())
