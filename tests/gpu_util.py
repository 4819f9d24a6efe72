"""Helpers shared by the GPU tests: move oracle results onto the device in
the library's layouts, and the output tolerances of the parity bound
(max |err| <= 2e-2 and cosine >= 0.9995 against the oracle)."""
import numpy as np
import torch

import oracle as O

MAX_ABS = 2e-2
MIN_COS = 0.9995


def lib():
    from quantized_attention_05_b200 import build
    build.build()
    import quantized_attention_05_b200 as S
    S.lib()
    return S


def qkv_from_oracle(S, oz, device="cuda", with_qdk=True):
    """QuantizedQKV on the device holding the ORACLE's codes and scales."""
    t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to(dt).to(device)  # noqa: E731
    qdk = t(oz["q_dot_kmean"].astype(np.float32), torch.float32) if with_qdk else None
    return S.QuantizedQKV(
        q=t(oz["q"], torch.int8), q_scale=t(oz["q_scale"], torch.float32),
        k=t(oz["k"], torch.int8), k_scale=t(oz["k_scale"], torch.float32),
        k_mean=t(oz["k_mean"], torch.float32), v=t(np.swapaxes(oz["v_t"], -1, -2), torch.uint8),
        v_scale=t(oz["v_scale"], torch.float32), q_dot_kmean=qdk,
        B=oz["B"], Hq=oz["Hq"], Hkv=oz["Hkv"], Nq=oz["Nq"], Nk=oz["Nk"], D=oz["D"])


def assert_attention_close(out_gpu, lse_gpu, ref, rows=None, what=""):
    """Compare device outputs with the oracle's (bf16-rounded out, lse)."""
    rows = ref["rows"] if rows is None else rows
    o = out_gpu.float().cpu().numpy().astype(np.float64)[:, :, rows]
    r = ref["out"]
    sel = ~np.isnan(r[..., 0])                        # heads the oracle computed
    og, rg = o[sel], r[sel]
    err = np.abs(og - rg).max()
    cos = O.cosine(og, rg)
    assert err <= MAX_ABS and cos >= MIN_COS, f"{what}: out max|err|={err:.3g} cos={cos:.6f}"
    if lse_gpu is not None:
        lg = lse_gpu.cpu().numpy().astype(np.float64)[:, :, rows][sel]
        lr = ref["lse"][sel]
        inf_r, inf_g = np.isneginf(lr), np.isneginf(lg)
        assert np.array_equal(inf_r, inf_g), f"{what}: -inf pattern of lse differs"
        fin = ~inf_r
        if fin.any():
            e = np.abs(lg[fin] - lr[fin]).max()
            c = O.cosine(lg[fin], lr[fin])
            assert e <= MAX_ABS and c >= MIN_COS, f"{what}: lse max|err|={e:.3g} cos={c:.6f}"
    return err, cos
