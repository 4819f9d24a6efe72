"""sage_quantize_qkv_noalloc: the quantiser for callers that cannot
allocate device memory (a plugin in a framework that owns every device
allocation, or a loop where a cudaMalloc is not allowed).  It keeps its
scratch in a fixed array inside the library instead of a caller workspace.

Checked through the C ABI: two calls in a row must give exactly what the
workspace entry point sage_quantize_qkv gives (the quantiser's outputs are
compared bit for bit, as in the other quantiser tests), and sizes whose
scratch would not fit the fixed array are refused before anything runs.
This file is collected last so that a failure here leaves every other test
already run."""
import ctypes

import numpy as np
import pytest
import torch

import workloads as W
from gpu_util import lib

pytestmark = pytest.mark.gpu

FIELDS = ("q", "q_scale", "k", "k_scale", "k_mean", "v", "v_scale", "q_dot_kmean")


def _call_noalloc(S, q, k, v, out):
    tq, tk, tv = S._as_tensor(q), S._as_tensor(k), S._as_tensor(v)
    s = out.struct()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return S.lib().sage_quantize_qkv_noalloc(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv),
                                             1, ctypes.byref(s), stream)


@pytest.mark.parametrize("w", [W.TINY.scaled(B=2, Hq=4, Hkv=2, N=300, D=128, seed=41),
                               W.CAUSAL_GQA.scaled(B=1, N=4096)],
                         ids=lambda w: f"{w.B}x{w.Hq}x{w.Hkv}x{w.N}x{w.D}")
def test_noalloc_matches_workspace_entry_point_twice(w):
    S = lib()
    q, k, v = (t.cuda() for t in W.make_qkv(w))
    ref = S.sage_quantize_qkv(q, k, v)
    torch.cuda.synchronize()
    for call in range(2):
        out = S.QuantizedQKV.empty(w.B, w.Hq, w.Hkv, w.N, w.N, w.D, q.device)
        st = _call_noalloc(S, q, k, v, out)
        assert st == S.SAGE_OK, f"call {call}: status {st}"
        torch.cuda.synchronize()
        for f in FIELDS:
            a, b = getattr(out, f).cpu().numpy(), getattr(ref, f).cpu().numpy()
            np.testing.assert_array_equal(a, b, err_msg=f"call {call}: {f}")
    st, site = S.sage_get_device_status()
    assert st == S.SAGE_OK


def test_noalloc_refuses_sizes_beyond_its_scratch():
    S = lib()
    B, H, N, D = 64, 64, 256, 128            # 4096 KV heads: scratch would exceed 4 MiB
    assert S.lib().sage_quantize_workspace_bytes(B, H, N, D) > 4 << 20
    fake = S.SageTensor(256, 0, B, H, N, D, H * N * D, N * D, D)
    z = S.SageQkvI8F8(256, 256, 256, 256, 256, 256, 256, 256, B, H, H, N, N, D)
    st = S.lib().sage_quantize_qkv_noalloc(ctypes.byref(fake), ctypes.byref(fake),
                                           ctypes.byref(fake), 1, ctypes.byref(z), None)
    assert st == S.SAGE_ERR_WORKSPACE
