"""The C ABI without a GPU: the library loads, exports every function the
header declares, the ctypes structs match the C layout, and host-side
validation rejects bad arguments before anything touches CUDA."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

import quantized_attention_05_b200 as S
from quantized_attention_05_b200 import build as B


@pytest.fixture(scope="module")
def L():
    B.build()
    return S.lib()


def declared_functions():
    text = open(S.HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sage_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 12
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing
    out = subprocess.run(["nm", "-D", "--defined-only", S.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (sage_[a-z0-9_]+)$", out, flags=re.M))
    assert set(names) <= exported


def test_library_has_no_driver_dependency_at_load():
    out = subprocess.run(["ldd", S.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out and "libcudart" not in out


def test_ctypes_layout_matches_header(tmp_path):
    src = tmp_path / "probe.c"
    src.write_text("""
#include <stdio.h>
#include <stddef.h>
#include "sage_b200.h"
int main(void) {
  printf("%zu %zu %zu %zu\\n", sizeof(sage_tensor), sizeof(sage_mask), sizeof(sage_qkv_i8f8),
         sizeof(sage_qkv_nvfp4));
  printf("%zu %zu %zu %zu\\n", offsetof(sage_tensor, B), offsetof(sage_mask, sq),
         offsetof(sage_qkv_i8f8, D), offsetof(sage_qkv_nvfp4, per_block_mean));
  return 0;
}""")
    exe = tmp_path / "probe"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.dirname(S.HEADER_PATH), str(src), "-o", str(exe)],
                   check=True)
    lines = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    sizes = list(map(int, lines[0].split()))
    offs = list(map(int, lines[1].split()))
    assert sizes == [ctypes.sizeof(S.SageTensor), ctypes.sizeof(S.SageMask), ctypes.sizeof(S.SageQkvI8F8),
                     ctypes.sizeof(S.SageQkvNvfp4)]
    assert offs == [S.SageTensor.B.offset, S.SageMask.sq.offset, S.SageQkvI8F8.D.offset,
                    S.SageQkvNvfp4.per_block_mean.offset]


def test_status_strings_and_version(L):
    assert L.sage_status_str(0) == b"ok"
    assert b"workspace" in L.sage_status_str(3)
    assert b"sm_100a" in L.sage_version()


def _t(ptr=16, dtype=0, B=1, H=2, N=256, D=64, sb=None, sh=None, sn=None):
    sn = D if sn is None else sn
    sh = N * sn if sh is None else sh
    sb = H * sh if sb is None else sb
    return S.SageTensor(ptr, dtype, B, H, N, D, sb, sh, sn)


def _q(ptr=256, B=1, Hq=2, Hkv=2, Nq=256, Nk=256, D=64):
    return S.SageQkvI8F8(ptr, ptr, ptr, ptr, ptr, ptr, ptr, ptr, B, Hq, Hkv, Nq, Nk, D)


def test_quantize_rejects_bad_arguments_on_host(L):
    byref = ctypes.byref
    out = _q()
    call = lambda q, k, v, o=out, ws=256, nb=1 << 20: L.sage_quantize_qkv(  # noqa: E731
        byref(q), byref(k), byref(v), 1, byref(o), ws, nb, None)
    assert call(_t(ptr=0), _t(), _t()) == S.SAGE_ERR_INVALID_ARG          # null pointer
    assert call(_t(ptr=8), _t(), _t()) == S.SAGE_ERR_INVALID_ARG          # misaligned
    assert call(_t(D=96), _t(D=96), _t(D=96)) == S.SAGE_ERR_UNSUPPORTED   # head_dim 96
    assert call(_t(dtype=7), _t(), _t()) == S.SAGE_ERR_INVALID_ARG        # dtype
    assert call(_t(), _t(dtype=1), _t()) == S.SAGE_ERR_INVALID_ARG        # mixed dtypes
    assert call(_t(H=3), _t(H=2), _t(H=2), _q(Hq=3)) == S.SAGE_ERR_INVALID_ARG   # Hq % Hkv
    assert call(_t(sn=60), _t(), _t()) == S.SAGE_ERR_INVALID_ARG          # stride not 16-byte rows
    assert call(_t(), _t(), _t(), _q(Nk=300)) == S.SAGE_ERR_INVALID_ARG   # out shape mismatch
    assert call(_t(), _t(), _t(), ws=0) == S.SAGE_ERR_INVALID_ARG         # no workspace
    assert call(_t(), _t(), _t(), nb=16) == S.SAGE_ERR_WORKSPACE          # workspace too small
    assert call(_t(H=4097), _t(H=1), _t(H=1), _q(Hq=4097, Hkv=1)) == S.SAGE_ERR_INVALID_ARG  # heads
    n1 = 128 * 2048 + 1                                                   # one key past the longest
    assert call(_t(), _t(N=n1), _t(N=n1), _q(Nk=n1)) == S.SAGE_ERR_UNSUPPORTED


def test_attention_rejects_bad_arguments_on_host(L):
    byref = ctypes.byref
    z = _q()
    f = L.sage_attn_fwd_quantized
    assert f(byref(z), 0, 0.0, 1, None, 256, 0, 2 * 256 * 64, 256 * 64, 64, None, None, 0, None) \
        == S.SAGE_ERR_INVALID_ARG                                   # return_lse without lse
    zz = _q()
    zz.q_dot_kmean = None
    assert f(byref(zz), 0, 0.0, 1, None, 256, 0, 0, 256 * 64, 64, 512, None, 0, None) \
        == S.SAGE_ERR_INVALID_ARG                                   # LSE needs q_dot_kmean
    assert f(byref(z), 0, 0.0, 0, None, 8, 0, 0, 256 * 64, 64, None, None, 0, None) \
        == S.SAGE_ERR_INVALID_ARG                                   # misaligned out
    assert f(byref(z), 0, 0.0, 0, None, 256, 5, 0, 256 * 64, 64, None, None, 0, None) \
        == S.SAGE_ERR_INVALID_ARG                                   # out dtype
    assert f(byref(z), 0, float("nan"), 0, None, 256, 0, 0, 256 * 64, 64, None, None, 0, None) \
        == S.SAGE_ERR_INVALID_ARG                                   # sm_scale
    m = S.SageMask(256, 1, 1, 256, 128, 0, 0, 256)                  # wrong key length
    assert f(byref(z), 0, 0.0, 0, byref(m), 256, 0, 0, 256 * 64, 64, None, 256, 1 << 20, None) \
        == S.SAGE_ERR_INVALID_ARG
    m = S.SageMask(256, 1, 1, 256, 256, 0, 0, 256)
    assert f(byref(z), 0, 0.0, 0, byref(m), 256, 0, 0, 256 * 64, 64, None, 256, 1, None) \
        == S.SAGE_ERR_WORKSPACE
    zbig = _q(Nq=128 * 4096, Nk=128 * 4096)
    assert f(byref(zbig), 0, 0.0, 0, None, 256, 0, 0, 256 * 64, 64, None, None, 0, None) \
        == S.SAGE_ERR_UNSUPPORTED
    zlong = _q(Nk=128 * 2048 + 1)                                   # one key past the longest
    assert f(byref(zlong), 0, 0.0, 0, None, 256, 0, 0, 256 * 64, 64, None, None, 0, None) \
        == S.SAGE_ERR_UNSUPPORTED


def test_fused_call_checks_num_kv_heads_and_workspace(L):
    byref = ctypes.byref
    q, k, v = _t(H=4), _t(H=2), _t(H=2)
    f = L.sage_attn_fwd
    assert f(byref(q), byref(k), byref(v), 0, 0.0, 3, 0, 1, None, 256, 0, 0, 64, None, 256, 1 << 30,
             None) == S.SAGE_ERR_INVALID_ARG                        # num_kv_heads != k.H
    need = L.sage_attn_fwd_workspace_bytes(1, 4, 2, 256, 256, 64, None)
    assert f(byref(q), byref(k), byref(v), 0, 0.0, 2, 0, 1, None, 256, 0, 0, 64, None, 256, need - 1,
             None) == S.SAGE_ERR_WORKSPACE


def test_workspace_sizes_cover_the_quantised_tensors(L):
    B_, Hq, Hkv, N, D = 4, 32, 8, 16384, 128
    need = L.sage_attn_fwd_workspace_bytes(B_, Hq, Hkv, N, N, D, None)
    payload = B_ * Hq * N * D + 2 * B_ * Hkv * N * D + B_ * Hq * N * 4
    assert payload < need < payload * 1.1
    assert L.sage_quantize_workspace_bytes(B_, Hkv, N, D) > 0
    assert L.sage_quantize_workspace_bytes(0, Hkv, N, D) == 0


def test_nvfp4_rejects_bad_arguments_on_host(L):
    byref = ctypes.byref
    q, k, v = _t(H=2), _t(H=2), _t(H=2)
    z = S.SageQkvNvfp4(256, 256, 256, 256, 256, 256, 256, 256, 256, 256, 1, 2, 2, 256, 256, 64, 256, 1)
    f = L.sage_quantize_qkv_nvfp4
    assert f(byref(q), byref(k), byref(v), 1, 300, byref(z), 256, 1 << 30, None) \
        == S.SAGE_ERR_INVALID_ARG                                   # unpadded length > N
    assert f(byref(q), byref(k), byref(v), 0, 256, byref(z), 256, 1 << 30, None) \
        == S.SAGE_ERR_INVALID_ARG                                   # per_block_mean mismatch
    need = L.sage_quantize_nvfp4_workspace_bytes(1, 2, 2, 256, 256, 64)
    assert f(byref(q), byref(k), byref(v), 1, 256, byref(z), 256, need - 1, None) == S.SAGE_ERR_WORKSPACE
    a = L.sage_attn_fwd_nvfp4
    assert a(byref(z), 0.0, 0, 0, 1, 256, 0, 0, 256 * 64, 64, 512, None) \
        == S.SAGE_ERR_INVALID_ARG                                   # per_block_mean mismatch
    zz = S.SageQkvNvfp4(256, 256, 256, 256, 256, 256, 256, 256, 256, None, 1, 2, 2, 256, 256, 64, 256, 1)
    assert a(byref(zz), 0.0, 0, 1, 1, 256, 0, 0, 256 * 64, 64, 512, None) \
        == S.SAGE_ERR_INVALID_ARG                                   # LSE without q_dot_kmean


def test_varlen_rejects_bad_arguments_on_host(L):
    byref = ctypes.byref
    pq = _t(B=1, H=4, N=1000, D=64, sn=4 * 64, sh=64)
    pk = _t(B=1, H=2, N=900, D=64, sn=2 * 64, sh=64)
    f = L.sage_attn_fwd_varlen
    need = L.sage_attn_fwd_varlen_workspace_bytes(3, 4, 2, 1000, 900, 512, 512, 64, 1)
    assert need > 0
    ok = dict(cu_q=256, cu_k=256, nseq=3, mq=512, mk=512, out=256, sn=4 * 64, sh=64, lse=512,
              ws=256, nb=need)

    def call(q=pq, k=pk, v=pk, **kw):
        a = dict(ok, **kw)
        return f(byref(q), byref(k), byref(v), a["cu_q"], a["cu_k"], a["nseq"], a["mq"], a["mk"], 0,
                 0.0, 1, 1, a["out"], a["sn"], a["sh"], a["lse"], a["ws"], a["nb"], None)
    assert call(q=_t(B=2, H=4, N=1000, D=64)) == S.SAGE_ERR_INVALID_ARG      # not packed (B=2)
    assert call(cu_q=0) == S.SAGE_ERR_INVALID_ARG                            # no cu_seqlens_q
    assert call(cu_k=258) == S.SAGE_ERR_INVALID_ARG                          # misaligned cu_seqlens_k
    assert call(nseq=0) == S.SAGE_ERR_INVALID_ARG
    assert call(mq=0) == S.SAGE_ERR_INVALID_ARG
    assert call(mk=128 * 4096) == S.SAGE_ERR_UNSUPPORTED                     # longer than supported
    assert call(lse=0) == S.SAGE_ERR_INVALID_ARG                             # return_lse without lse
    assert call(sn=60) == S.SAGE_ERR_INVALID_ARG                             # out stride
    assert call(nb=need - 1) == S.SAGE_ERR_WORKSPACE
    assert call(q=_t(B=1, H=3, N=1000, D=64)) == S.SAGE_ERR_INVALID_ARG      # Hq % Hkv
    assert call(q=_t(B=1, H=4, N=1000, D=96), k=_t(B=1, H=2, N=900, D=96),
                v=_t(B=1, H=2, N=900, D=96)) == S.SAGE_ERR_UNSUPPORTED      # head_dim 96
    assert L.sage_attn_fwd_varlen_workspace_bytes(0, 4, 2, 1000, 900, 512, 512, 64, 1) == 0


def test_host_call_rejects_bad_arguments_on_host(L):
    byref = ctypes.byref
    q, k, v = _t(H=4), _t(H=2), _t(H=2)
    f = L.sage_attn_fwd_host
    need = L.sage_attn_fwd_host_workspace_bytes(1, 4, 2, 256, 256, 64, None, 0)
    assert need > 0
    ok = dict(q=q, k=k, v=v, nkv=2, lse_flag=1, out=256, sn=64, sh=256 * 64, lse=512, chunk=0,
              ws=256, nb=need)

    def call(**kw):
        a = dict(ok, **kw)
        return f(byref(a["q"]), byref(a["k"]), byref(a["v"]), 1, 0.0, a["nkv"], a["lse_flag"], 1, None,
                 a["out"], 4 * 256 * 64, a["sh"], a["sn"], a["lse"], a["chunk"], a["ws"], a["nb"], None)
    assert call(nkv=3) == S.SAGE_ERR_INVALID_ARG                     # num_kv_heads != k.H
    assert call(k=_t(H=2, dtype=1)) == S.SAGE_ERR_INVALID_ARG        # k dtype differs from q
    assert call(v=_t(H=2, N=128)) == S.SAGE_ERR_INVALID_ARG          # v length differs from k
    assert call(lse=0) == S.SAGE_ERR_INVALID_ARG                     # return_lse without lse
    assert call(out=0) == S.SAGE_ERR_INVALID_ARG
    assert call(sn=60) == S.SAGE_ERR_INVALID_ARG                     # out token stride
    assert call(chunk=-1) == S.SAGE_ERR_INVALID_ARG
    assert call(ws=0) == S.SAGE_ERR_INVALID_ARG
    assert call(ws=384) == S.SAGE_ERR_INVALID_ARG                    # workspace not 256-aligned
    assert call(nb=need - 1) == S.SAGE_ERR_WORKSPACE
    assert call(q=_t(H=4, D=96), k=_t(H=2, D=96), v=_t(H=2, D=96)) == S.SAGE_ERR_UNSUPPORTED
    assert L.sage_attn_fwd_host_workspace_bytes(1, 4, 2, 256, 256, 64, None, -1) == 0
    assert L.sage_attn_fwd_host_workspace_bytes(1, 3, 2, 256, 256, 64, None, 0) == 0


def test_host_call_workspace_is_three_chunk_slots_plus_one_chunk_workspace(L):
    B_, Hq, Hkv, N, D = 4, 32, 8, 16384, 128
    G = Hq // Hkv
    # automatic chunk: the number of KV-head groups nearest to 100 MB of bf16 inputs (4 here)
    per_group_in = (G * N + 2 * N) * D * 2
    gpc = max(1, ((100 << 20) + per_group_in // 2) // per_group_in)
    assert gpc == 4
    slot = gpc * (G * N * D * 2 + 2 * N * D * 2 + G * N * D * 2 + G * N * 4)
    one_chunk = L.sage_attn_fwd_workspace_bytes(1, gpc * G, gpc, N, N, D, None)
    need = L.sage_attn_fwd_host_workspace_bytes(B_, Hq, Hkv, N, N, D, None, 0)
    assert need == pytest.approx(3 * slot + one_chunk, abs=3 * 5 * 256)
    # explicit chunking, with a smaller last chunk per batch entry (8 = 3 + 3 + 2)
    need3 = L.sage_attn_fwd_host_workspace_bytes(B_, Hq, Hkv, N, N, D, None, 3)
    assert need3 == pytest.approx(3 * slot * 3 // 4 + L.sage_attn_fwd_workspace_bytes(
        1, 3 * G, 3, N, N, D, None), abs=3 * 5 * 256 + 4096)
    # one chunk of everything when the chunk size exceeds the heads
    assert L.sage_attn_fwd_host_workspace_bytes(1, 4, 2, 256, 256, 64, None, 99) == \
        L.sage_attn_fwd_host_workspace_bytes(1, 4, 2, 256, 256, 64, None, 2)


def test_nvfp4_host_call_rejects_bad_arguments_on_host(L):
    byref = ctypes.byref
    q, k, v = _t(H=4), _t(H=2), _t(H=2)
    f = L.sage_attn_fwd_nvfp4_host
    need = L.sage_attn_fwd_nvfp4_host_workspace_bytes(1, 4, 2, 256, 256, 64, 0)
    assert need > L.sage_attn_fwd_host_workspace_bytes(1, 4, 2, 256, 256, 64, None, 0) // 4
    ok = dict(q=q, k=k, v=v, ukl=0, lse_flag=1, out=256, sn=64, lse=512, chunk=0, ws=256, nb=need)

    def call(**kw):
        a = dict(ok, **kw)
        return f(byref(a["q"]), byref(a["k"]), byref(a["v"]), 0.0, 0, 1, a["ukl"], a["lse_flag"],
                 a["out"], 4 * 256 * 64, 256 * 64, a["sn"], a["lse"], a["chunk"], a["ws"], a["nb"], None)
    assert call(ukl=257) == S.SAGE_ERR_INVALID_ARG                   # unpadded length > Nk
    assert call(k=_t(H=2, dtype=1)) == S.SAGE_ERR_INVALID_ARG        # dtype differs from q
    assert call(q=_t(H=3)) == S.SAGE_ERR_INVALID_ARG                 # Hq % Hkv
    assert call(lse=0) == S.SAGE_ERR_INVALID_ARG
    assert call(sn=60) == S.SAGE_ERR_INVALID_ARG
    assert call(chunk=-2) == S.SAGE_ERR_INVALID_ARG
    assert call(ws=384) == S.SAGE_ERR_INVALID_ARG
    assert call(nb=need - 1) == S.SAGE_ERR_WORKSPACE
    assert L.sage_attn_fwd_nvfp4_host_workspace_bytes(1, 4, 2, 256, 256, 64, -1) == 0


def test_calls_without_queries_return_ok_without_touching_the_device(L):
    """B == 0 or Nq == 0: the whole-path calls check the sizes, look at no
    pointer (null here, as for empty tensors) and return SAGE_OK; no CUDA
    call is made, which is what lets this run on a machine without a GPU."""
    byref = ctypes.byref

    def fused(q, k, v, nkv=2):
        return L.sage_attn_fwd(byref(q), byref(k), byref(v), 1, 0.0, nkv, 1, 1, None,
                               None, 0, 0, 64, None, None, 0, None)

    def host(q, k, v, nkv=2):
        return L.sage_attn_fwd_host(byref(q), byref(k), byref(v), 1, 0.0, nkv, 1, 1, None,
                                    None, 0, 0, 64, None, 0, None, 0, None)

    def nvfp4(q, k, v, ukl=0):
        return L.sage_attn_fwd_nvfp4_host(byref(q), byref(k), byref(v), 0.0, 1, 1, ukl, 1,
                                          None, 0, 0, 64, None, 0, None, 0, None)

    for f in (fused, host, nvfp4):
        assert f(_t(ptr=0, H=4, N=0), _t(ptr=0), _t(ptr=0)) == S.SAGE_OK              # no queries
        assert f(_t(ptr=0, B=0, H=4), _t(ptr=0, B=0), _t(ptr=0, B=0)) == S.SAGE_OK     # no batch
        assert f(_t(ptr=0, H=4, N=0), _t(ptr=0, N=0), _t(ptr=0, N=0)) == S.SAGE_OK     # no keys either
        assert f(_t(ptr=0, H=3, N=0), _t(ptr=0), _t(ptr=0)) == S.SAGE_ERR_INVALID_ARG  # Hq % Hkv
        assert f(_t(ptr=0, H=4, N=0), _t(ptr=0, dtype=1), _t(ptr=0)) == S.SAGE_ERR_INVALID_ARG
        assert f(_t(ptr=0, H=4, N=0), _t(ptr=0), _t(ptr=0, N=128)) == S.SAGE_ERR_INVALID_ARG
        assert f(_t(ptr=0, B=0, H=4), _t(ptr=0), _t(ptr=0)) == S.SAGE_ERR_INVALID_ARG  # batch mismatch
        assert f(_t(ptr=0, H=4, N=0, D=96), _t(ptr=0, D=96), _t(ptr=0, D=96)) == S.SAGE_ERR_UNSUPPORTED
        # keys are required when there are queries
        assert f(_t(H=4), _t(N=0), _t(N=0)) == S.SAGE_ERR_INVALID_ARG
    assert fused(_t(ptr=0, H=4, N=0), _t(ptr=0), _t(ptr=0), nkv=1) == S.SAGE_ERR_INVALID_ARG
    assert host(_t(ptr=0, H=4, N=0), _t(ptr=0), _t(ptr=0), nkv=1) == S.SAGE_ERR_INVALID_ARG
    assert nvfp4(_t(ptr=0, H=4, N=0), _t(ptr=0), _t(ptr=0), ukl=257) == S.SAGE_ERR_INVALID_ARG


def test_device_calls_refuse_more_head_pairs_than_a_grid_holds(L):
    """More than 65535 (batch entry, Q head) pairs in one device call --
    (sequence, KV head) pairs in a varlen call -- is SAGE_ERR_UNSUPPORTED,
    found on the host before anything is enqueued; the host-buffer call,
    which works one chunk of heads at a time, is not bound by it."""
    byref = ctypes.byref
    q, k = _t(B=64, H=1025, N=128), _t(B=64, H=1, N=128)          # 65600 pairs
    assert L.sage_attn_fwd(byref(q), byref(k), byref(k), 0, 0.0, 1, 0, 1, None, 256, 0, 0, 64,
                           None, 256, 1 << 40, None) == S.SAGE_ERR_UNSUPPORTED
    z = _q(B=64, Hq=1025, Hkv=1, Nq=128, Nk=128)
    assert L.sage_quantize_qkv(byref(q), byref(k), byref(k), 1, byref(z), 256, 1 << 40,
                               None) == S.SAGE_ERR_UNSUPPORTED
    assert L.sage_attn_fwd_quantized(byref(z), 0, 0.0, 0, None, 256, 0, 0, 128 * 64, 64, None, 256,
                                     1 << 40, None) == S.SAGE_ERR_UNSUPPORTED
    # 65472 pairs pass the size checks: the next check (a mask of the wrong
    # key length) is the one that answers
    zz = _q(B=64, Hq=1023, Hkv=1, Nq=128, Nk=128)
    bad_mask = S.SageMask(256, 1, 1, 128, 64, 0, 0, 128)
    assert L.sage_attn_fwd_quantized(byref(zz), 0, 0.0, 0, byref(bad_mask), 256, 0, 0, 128 * 64, 64,
                                     None, 256, 1 << 40, None) == S.SAGE_ERR_INVALID_ARG
    assert L.sage_attn_fwd_host_workspace_bytes(64, 1025, 1, 128, 128, 64, None, 0) > 0
    pq, pk = _t(H=4, N=1 << 20), _t(H=1, N=1 << 20)                # packed: 65600 sequences x 1 KV head
    assert L.sage_attn_fwd_varlen(byref(pq), byref(pk), byref(pk), 256, 256, 65600, 16, 16, 0, 0.0,
                                  1, 0, 256, 64, 64, None, 256, 1 << 40, None) == S.SAGE_ERR_UNSUPPORTED
