"""The Python binding's marshalling on the host (CPU tensors; no library call is reached).

The binding only turns torch tensors into ssm_scan_params (sizes, strides, pointers, flags)
and rejects layouts the C ABI cannot express; these checks run before any call into the
library, so CPU tensors exercise them without a GPU.
"""
import pytest

torch = pytest.importorskip("torch")

import selective_state_space_15_b200 as ssm  # noqa: E402


def _batch(b=2, D=6, N=16, L=40, dtype=torch.bfloat16, G=None):
    x = lambda: torch.zeros(b, D, L, dtype=dtype)  # noqa: E731
    shape_bc = (b, G, N, L) if G else (b, N, L)
    return dict(u=x(), delta=x(), z=x(), B=torch.zeros(shape_bc, dtype=dtype), C=torch.zeros(shape_bc, dtype=dtype),
                A=torch.zeros(D, N), Dskip=torch.zeros(D), delta_bias=torch.zeros(D))


def test_scan_params_fields():
    t = _batch()
    y = torch.zeros(2, 6, 40, dtype=torch.float32)
    p = ssm.scan_params(t["u"], t["delta"], t["B"], t["C"], t["A"], t["Dskip"], t["delta_bias"], t["z"], y=y, zoh=True)
    assert (p.dtype, p.y_fp32, p.batch, p.dim, p.dstate, p.seqlen) == (ssm.SSM_BF16, 1, 2, 6, 16, 40)
    assert (p.x_batch_stride, p.x_dim_stride, p.bc_batch_stride, p.bc_state_stride) == (240, 40, 640, 40)
    assert p.discretization == ssm.DISC_ZOH and p.ngroups == 0
    assert p.u == t["u"].data_ptr() and p.C == t["C"].data_ptr() and p.h0 is None
    assert ssm.scan_params(t["u"], t["delta"], t["B"], t["C"], t["A"]).discretization == ssm.DISC_EULER


def test_scan_params_channel_groups_and_padded_rows():
    t = _batch(D=6, G=3)
    p = ssm.scan_params(t["u"], t["delta"], t["B"], t["C"], t["A"])
    assert (p.ngroups, p.bc_group_stride, p.bc_batch_stride) == (3, 16 * 40, 3 * 16 * 40)
    # rows padded beyond the sequence (a view of a wider buffer): strides pass through
    wide = torch.zeros(2, 6, 48, dtype=torch.bfloat16)
    u = wide[:, :, :40]
    p = ssm.scan_params(u, u, t["B"][:, 0], t["C"][:, 0], t["A"])
    assert (p.x_batch_stride, p.x_dim_stride, p.seqlen) == (288, 48, 40)


@pytest.mark.parametrize("bad", ["time_stride", "delta_shape", "bc_shape", "bc_strides", "A_dtype", "A_layout",
                                 "y_dtype", "u_dtype"])
def test_scan_params_rejects_bad_layouts(bad):
    t = _batch()
    y = None
    if bad == "time_stride":
        t["u"] = torch.zeros(2, 40, 6, dtype=torch.bfloat16).transpose(1, 2)
    elif bad == "delta_shape":
        t["delta"] = torch.zeros(2, 6, 39, dtype=torch.bfloat16)
    elif bad == "bc_shape":
        t["B"] = torch.zeros(2, 8, 40, dtype=torch.bfloat16)
    elif bad == "bc_strides":
        t["C"] = torch.zeros(2, 16, 48, dtype=torch.bfloat16)[:, :, :40]
    elif bad == "A_dtype":
        t["A"] = torch.zeros(6, 16, dtype=torch.float64)
    elif bad == "A_layout":
        t["A"] = torch.zeros(16, 6).t()
    elif bad == "y_dtype":
        y = torch.zeros(2, 6, 40, dtype=torch.float16)
    elif bad == "u_dtype":
        for k in ("u", "delta", "z"):
            t[k] = t[k].to(torch.float16)
    with pytest.raises((ValueError, TypeError)):
        ssm.scan_params(t["u"], t["delta"], t["B"], t["C"], t["A"], t["Dskip"], t["delta_bias"], t["z"], y=y)


def test_varlen_params_fields_and_checks():
    D, N, T, W = 5, 16, 30, 32
    u = torch.zeros(D, W, dtype=torch.bfloat16)
    B = torch.zeros(N, W, dtype=torch.bfloat16)
    A = torch.zeros(D, N)
    p = ssm.varlen_params(u, u, B, B, A, total=T, zoh=True)
    assert (p.batch, p.dim, p.dstate, p.seqlen, p.x_dim_stride, p.bc_state_stride) == (1, D, N, T, W, W)
    assert p.discretization == ssm.DISC_ZOH
    with pytest.raises(ValueError):
        ssm.varlen_params(u, u, torch.zeros(N, 20, dtype=torch.bfloat16), torch.zeros(N, 20, dtype=torch.bfloat16),
                          A, total=T)   # B shorter than the packed tokens
    cu = torch.tensor([0, 10, 30], dtype=torch.int64)
    with pytest.raises(ValueError):
        ssm.scan_fwd_varlen(u, u, B, B, A, cu, total=T)   # cu_seqlens must be int32


def test_pool_and_decode_argument_checks():
    D, N, S = 5, 16, 4
    pool = torch.zeros(S, D, N)
    u = torch.zeros(3, D, dtype=torch.bfloat16)
    B = torch.zeros(3, N, dtype=torch.bfloat16)
    A = torch.zeros(D, N)
    with pytest.raises(ValueError):
        ssm.state_update(pool, torch.zeros(3, dtype=torch.int64), u, u, B, B, A)   # slot ids must be int32
    C_padded = torch.zeros(3, 32, dtype=torch.bfloat16)[:, :N]   # row stride differs from B's
    with pytest.raises(ValueError):
        ssm.state_update(pool, torch.zeros(3, dtype=torch.int32), u, u, B, C_padded, A)
    cu = torch.tensor([0, 2, 3], dtype=torch.int32)
    uu = torch.zeros(D, 8, dtype=torch.bfloat16)
    BB = torch.zeros(N, 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        ssm.scan_fwd_varlen_pool(uu, uu, BB, BB, A, cu, pool, torch.zeros(3, dtype=torch.int32), total=3)  # 2 seqs
    with pytest.raises(ValueError):
        ssm.scan_fwd_varlen_pool(uu, uu, BB, BB, A, cu, torch.zeros(S, D + 1, N), torch.zeros(2, dtype=torch.int32),
                                 total=3)
