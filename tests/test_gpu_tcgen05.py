"""The tcgen05 building blocks in isolation, on codes made by the oracle:
the INT8 QK^T tile must equal the exact integer product bit for bit; the
FP8 PV tile must equal the exact product of the decoded E4M3 values up to
FP32 accumulation; a bounded wait that nobody releases must time out and
report its site without hanging the GPU."""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from gpu_util import lib, qkv_from_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    return lib()


@pytest.mark.parametrize("D", [64, 128])
def test_qk_int32_tile_bit_exact(S, D):
    w = W.TINY.scaled(B=2, Hq=4, Hkv=2, N=384, D=D, seed=21, k_offset_std=5.0)
    q, k, v = W.make_qkv(w)
    oz = O.quantize_qkv_i8f8(q, k, v)
    z = qkv_from_oracle(S, oz)
    for (b, h, qb, kb) in [(0, 0, 0, 0), (1, 3, 2, 1), (0, 2, 1, 2), (1, 1, 2, 2)]:
        tile = S.sage_debug_qk_int32(z, b, h, qb, kb).cpu().numpy()
        np.testing.assert_array_equal(tile, O.qk_int32_tile(oz, b, h, qb, kb), err_msg=f"{b,h,qb,kb}")


def test_qk_int32_extremes(S):
    """All codes +-127: |S| = 127*127*128 exercises the int32 accumulator."""
    B, H, N, D = 1, 1, 128, 128
    g = torch.Generator().manual_seed(5)
    sign = (torch.randint(0, 2, (B, H, N, D), generator=g) * 2 - 1).numpy()
    oz = dict(q=(127 * sign).astype(np.int8), k=(127 * np.ones_like(sign)).astype(np.int8),
              q_scale=np.ones((1, 1, 1), np.float32), k_scale=np.ones((1, 1, 1), np.float32),
              k_mean=np.zeros((1, 1, D), np.float32), v_t=np.zeros((1, 1, D, N), np.uint8),
              v_scale=np.ones((1, 1, D), np.float32), q_dot_kmean=np.zeros((1, 1, N)),
              B=B, Hq=H, Hkv=H, Nq=N, Nk=N, D=D)
    oz["k"][0, 0, 5] = -127
    z = qkv_from_oracle(S, oz)
    tile = S.sage_debug_qk_int32(z, 0, 0, 0, 0).cpu().numpy()
    np.testing.assert_array_equal(tile, O.qk_int32_tile(oz, 0, 0, 0, 0))


@pytest.mark.parametrize("D", [64, 128])
def test_pv_fp8_tile(S, D):
    w = W.TINY.scaled(B=1, Hq=2, Hkv=2, N=256, D=D, seed=22)
    q, k, v = W.make_qkv(w)
    oz = O.quantize_qkv_i8f8(q, k, v)
    z = qkv_from_oracle(S, oz)
    g = torch.Generator().manual_seed(7)
    p = torch.rand(128, 128, generator=g) * 448
    p[:, ::3] = 0
    p_codes = O.e4m3_encode(p.double().numpy())
    acc = S.sage_debug_pv_fp32(z, torch.from_numpy(p_codes).cuda(), 0, 1, 1).cpu().numpy()
    pdec = O.e4m3_decode(p_codes)
    vdec = O.e4m3_decode(oz["v_t"][0, 1, :, 128:256])        # [D, 128 keys]
    exact = pdec @ vdec.T                                    # [128, D]
    np.testing.assert_allclose(acc, exact, rtol=1e-5, atol=1e-5 * np.abs(exact).max())


def test_bounded_wait_times_out_and_reports(S):
    st, site = S.sage_get_device_status()
    assert st == S.SAGE_OK
    S.sage_debug_wait_timeout(2000)          # 2 ms bound on a barrier nobody releases
    st, site = S.sage_get_device_status()
    assert st == S.SAGE_ERR_TIMEOUT and site == 8
    st, site = S.sage_get_device_status()    # cleared, and the context is still usable
    assert st == S.SAGE_OK
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum()) == 8.0
