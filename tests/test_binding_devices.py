"""The binding's device checks, on a machine without a GPU: every device
call refuses host tensors and tensors spread over several GPUs before any
pointer reaches the library (a host pointer handed to a kernel would be an
invalid device address)."""
import dataclasses

import pytest
import torch

import quantized_attention_05_b200 as S


@dataclasses.dataclass
class _Fake:
    """Just the two attributes the check reads."""
    is_cuda: bool
    device: torch.device


def _cuda(i):
    return _Fake(True, torch.device("cuda", i))


def test_one_device_is_found_and_none_entries_are_skipped():
    assert S._cuda_device() is None
    assert S._cuda_device(None, None) is None
    assert S._cuda_device(_cuda(1), None, _cuda(1)) == torch.device("cuda", 1)


def test_host_tensors_and_mixed_devices_are_refused():
    with pytest.raises(ValueError, match="expected CUDA tensors"):
        S._cuda_device(_cuda(0), torch.zeros(1))
    with pytest.raises(ValueError, match="one CUDA device"):
        S._cuda_device(_cuda(0), None, _cuda(1))


def test_device_calls_refuse_host_tensors_before_the_library():
    q = torch.zeros(1, 2, 128, 64, dtype=torch.bfloat16)
    k = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    calls = [
        lambda: S.sage_attn_fwd(q, k, k),
        lambda: S.sage_quantize_qkv(q, k, k),
        lambda: S.sage_quantize_qkv_noalloc(q, k, k),
        lambda: S.sage_quantize_qkv_nvfp4(q, k, k),
        lambda: S.sage_attn_fwd_varlen(q[0].transpose(0, 1), k[0].transpose(0, 1), k[0].transpose(0, 1),
                                       torch.tensor([0, 128], dtype=torch.int32),
                                       torch.tensor([0, 128], dtype=torch.int32), 128, 128),
        lambda: S.sage_lse_merge(torch.zeros(1, 2, 128, 64), torch.zeros(1, 2, 128), q,
                                 torch.zeros(1, 2, 128)),
        lambda: S.sage_lse_merge_finalize(torch.zeros(1, 2, 128, 64), q.clone()),
    ]
    for call in calls:
        with pytest.raises(ValueError, match="expected CUDA tensors"):
            call()


def test_host_calls_refuse_a_host_workspace():
    q = torch.zeros(1, 2, 128, 64, dtype=torch.bfloat16)
    k = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    ws = torch.zeros(16, dtype=torch.uint8)
    out = torch.empty_like(q)
    with pytest.raises(ValueError, match="expected CUDA tensors"):
        S.sage_attn_fwd_host(q, k, k, out=out, ws=ws, device="cuda:0")
    with pytest.raises(ValueError, match="expected CUDA tensors"):
        S.sage_attn_fwd_nvfp4_host(q, k, k, out=out, ws=ws, device="cuda:0")
    with pytest.raises(ValueError, match="CUDA device"):
        S.sage_attn_fwd_host(q, k, k, out=out, device="cpu")
