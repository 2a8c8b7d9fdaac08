"""Shared helpers of the GPU parity tests: move seeded inputs to the device, run the C ABI through
the binding, bring results back as float64 numpy arrays, compare."""
import numpy as np

import ispa_inputs as inp


def torch_dtype(wl_or_name):
    import torch
    name = wl_or_name if isinstance(wl_or_name, str) else wl_or_name.dtype
    return torch.bfloat16 if name == "bf16" else torch.float32


def dev(x, dtype):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x)).to(device="cuda", dtype=dtype)


def host(t):
    import torch
    return t.detach().to(torch.float64).cpu().numpy()


def rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))


SEGS = ("q", "k_sink", "v_sink", "k_loc", "v_loc", "k_hist", "v_hist")


def run_attention(x, dtype, **kw):
    """Runs ispa_dual_stream_attn on the seeded inputs `x` (dict of [tokens, H, hd] arrays)."""
    import torch
    from kv_cache_compression_tma_b200 import ispa
    t = {k: dev(x[k], dtype) for k in SEGS}
    out = ispa.dual_stream_attn(t["q"], t["k_sink"], t["v_sink"], t["k_loc"], t["v_loc"], t["k_hist"], t["v_hist"],
                                **kw)
    torch.cuda.synchronize()
    return out


def attention_errors(out, ref, rows=None):
    """Errors of GPU attention outputs against the oracle's separate passes (optionally on rows)."""
    H = ref["lse_loc"].shape[0]
    n = ref["O_loc"].shape[0]
    o_loc = host(out["o_loc"])
    o_full = host(out["o_full"])
    lse_l = host(out["lse_loc"])
    lse_h = host(out["lse_hist"])
    if rows is not None:
        o_loc, o_full = o_loc[rows], o_full[rows]
        lse_l, lse_h = lse_l[:, rows], lse_h[:, rows]
    ref_loc = ref["O_loc"].reshape(n, -1)
    ref_full = ref["O_full"].reshape(n, -1)
    err = {"o_loc": rel(o_loc, ref_loc), "o_full": rel(o_full, ref_full),
           "lse_loc": float(np.max(np.abs(lse_l - ref["lse_loc"])))}
    # the post-hoc merge of the two GPU branches must give the oracle's separate full pass
    err["lse_full"] = float(np.max(np.abs(np.logaddexp(lse_l, lse_h) - ref["lse_full"])))
    if ref.get("with_hist", True):
        fin = np.isfinite(ref["lse_hist"])
        err["lse_hist"] = float(np.max(np.abs(lse_h[fin] - ref["lse_hist"][fin]))) if fin.any() else 0.0
        err["lse_hist_inf_ok"] = bool(np.all(np.isneginf(lse_h[~fin])))
    else:
        err["lse_hist_inf_ok"] = True
    if out.get("d") is not None:
        dd = host(out["d"])
        if rows is not None:
            dd = dd[rows]
        err["d"] = rel(dd, ref_full - ref_loc)
    return err


ATTN_TOL = {"o_loc": 1e-2, "o_full": 1e-2, "d": 1e-2, "lse_loc": 2e-3, "lse_hist": 2e-3, "lse_full": 2e-3}


def assert_attention_ok(err, tol=ATTN_TOL):
    for k, t in tol.items():
        if k in err:
            assert err[k] <= t, (k, err[k], err)
    assert err["lse_hist_inf_ok"], err
