"""Rotated key basis for models without QK-norm (Fathom, yeyulingfeng.com
article, section 基座选择): keys are stored as planes of their coordinates in
an eigenbasis of the calibration keys' covariance, ordered by each
direction's contribution to score variance, and queries are rotated to
match; all D rotated coordinates are kept, and the plan decides how deep
to read each one.

This is set-up work of the caller (done once per session, like sigma^2):
the scan itself only ever sees the rotated keys and queries.  The basis is
computed in fp64 with torch; the rotation of keys and queries is an fp32
matrix product.
"""
from __future__ import annotations

import torch


def klt_basis(cal_keys: torch.Tensor, q: torch.Tensor) -> torch.Tensor:
    """Per group, the orthonormal basis U [H][D][D] (columns = directions):
    eigenvectors u_i of the centred covariance of ``cal_keys`` [H][N][D],
    ordered by lambda_i * u_i^T Sigma_q u_i descending, where Sigma_q is the
    second moment of the group's queries ``q`` [H][G][D]."""
    x = cal_keys.to(torch.float64)
    x = x - x.mean(dim=1, keepdim=True)
    cov = x.transpose(1, 2) @ x / x.shape[1]
    lam, vec = torch.linalg.eigh(cov)                       # ascending eigenvalues
    qq = q.to(torch.float64)
    sq = qq.transpose(1, 2) @ qq                            # [H][D][D]
    weight = lam * torch.einsum("hdi,hde,hei->hi", vec, sq, vec)
    order = torch.argsort(weight, dim=1, descending=True)
    return torch.gather(vec, 2, order[:, None, :].expand_as(vec)).to(torch.float32)


def rotate(x: torch.Tensor, U: torch.Tensor) -> torch.Tensor:
    """Coordinates of rows of x [H][N][D] in the basis U [H][D][D] (fp32)."""
    return torch.bmm(x.to(torch.float32), U).contiguous()
