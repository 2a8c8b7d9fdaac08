"""FAST-AR TempCache on the GPU (FAST-AR page, section 2 "Core components", A, Lemma 5.1) against the
oracle's tempcache_match / tempcache_merge / biased_softmax_attention, through the C ABI.

* Matching is an argmax over floating-point similarities: where the oracle's best entry beats the
  runner-up by more than 1e-3 the GPU must pick the same entry; elsewhere (near-ties) its entry must
  score within 1e-3 of the best.  Similarities within 1e-3 (bf16 keys, fp32 accumulation vs fp64).
* The merge is checked on the kernel's own decisions (idx, sim): counts, slots and keys exactly,
  values within the bf16 rounding of a mean, bias = ln(count), inverse norms within fp32 rounding.
* Lemma 5.1: attention over a cache whose duplicated keys were merged (bias ln(size)) equals attention
  over the unmerged frames, within the bf16 attention tolerance (1e-2 relative Frobenius)."""
import math

import numpy as np
import pytest

import ispa_inputs as inp
from oracle import ispa_oracle as orc
from gpu_helpers import dev, host, rel

pytestmark = pytest.mark.gpu


def frames(n_frames, T, H, hd, seed, rho=0.9):
    """AR(1) K/V frames (the workloads' recipe), bf16-rounded, [n_frames, T, H, hd]."""
    wl = inp.Workload("tc", H, hd, T, T, 1, ((tuple(range(1, n_frames)), (n_frames,)),), 1, None, 1e-2, rho, 2.0,
                      "bf16")
    k = inp.round_bf16(inp.kv_timeline(wl, 0, "k", seed, n_frames=n_frames))
    v = inp.round_bf16(inp.kv_timeline(wl, 0, "v", seed, n_frames=n_frames))
    return k, v


def cache_state(tc):
    n = tc.n_cache
    return (host(tc.k[:n]), host(tc.v[:n]), tc.count[:, :n].cpu().numpy().astype(np.int64),
            tc.n_valid.cpu().numpy().astype(np.int64))


def check_match(k_new, k_cache, count, idx_gpu, sim_gpu):
    idx_o, sim_o = orc.tempcache_match(k_new, k_cache, count)
    T, H, _ = k_new.shape
    for h in range(H):
        valid = np.nonzero(count[h] > 0)[0]
        a, b = k_new[:, h].astype(np.float64), k_cache[valid, h].astype(np.float64)
        na, nb = np.linalg.norm(a, axis=1), np.linalg.norm(b, axis=1)
        cos = np.where((na[:, None] > 0) & (nb[None, :] > 0), (a @ b.T) / np.maximum(na[:, None] * nb[None, :], 1e-300), 0.0)
        srt = np.sort(cos, axis=1)
        gap = srt[:, -1] - srt[:, -2] if cos.shape[1] > 1 else np.full(T, np.inf)
        clear = gap > 1e-3
        assert np.array_equal(idx_gpu[h][clear], idx_o[h][clear]), h
        pos = np.minimum(np.searchsorted(valid, idx_gpu[h]), len(valid) - 1)
        assert np.all(valid[pos] == idx_gpu[h])                       # a live entry
        assert np.all(cos[np.arange(T), pos] >= srt[:, -1] - 1e-3)     # near-ties: as good as the best
        assert np.max(np.abs(sim_gpu[h] - sim_o[h])) <= 1e-3


def test_match_and_merge_against_oracle(cuda_ok):
    """Three frames of a 4-head, head_dim 128 cache (AR(1) rho 0.95, so frames are near-duplicates):
    every match and merge against the oracle, on the kernel's decisions."""
    import torch
    from kv_cache_compression_tma_b200 import ispa
    T, H, hd, theta = 300, 4, 128, 0.9
    k, v = frames(4, T, H, hd, seed=71, rho=0.95)
    tc = ispa.TempCache(H, hd, capacity=4 * T)
    for f in range(3):
        before = cache_state(tc)
        kn, vn = dev(k[f], torch.bfloat16), dev(v[f], torch.bfloat16)
        idx, sim = tc.match(kn)
        torch.cuda.synchronize()
        idx_g, sim_g = idx.cpu().numpy().astype(np.int64), sim.cpu().numpy().astype(np.float64)
        if f == 0:
            assert np.all(idx_g == -1) and np.all(np.isneginf(sim_g))
        else:
            check_match(k[f], before[0], before[2], idx_g, sim_g)
        tc.merge(kn, vn, idx, sim, theta)
        torch.cuda.synchronize()
        assert ispa.get_device_status() == ispa.ISPA_OK
        k_o, v_o, c_o = orc.tempcache_merge(before[0], before[1], before[2], k[f], v[f], idx_g, sim_g, theta)
        k_g, v_g, c_g, n_g = cache_state(tc)
        assert np.array_equal(c_g, c_o)
        assert np.array_equal(n_g, np.count_nonzero(c_o, axis=1))
        assert np.array_equal(k_g, k_o)
        assert rel(v_g, v_o) <= 4e-3 and np.max(np.abs(v_g - v_o)) <= 2.0 ** -7 * np.max(np.abs(v_o))
        bias = tc.bias[:, :tc.n_cache].cpu().numpy()
        with np.errstate(divide="ignore"):
            want = np.log(c_o.astype(np.float64))
        assert np.array_equal(np.isneginf(bias), np.isneginf(want))
        fin = np.isfinite(want)
        assert np.max(np.abs(bias[fin] - want[fin])) <= 1e-6
        inv = tc.inv_norm[:, :tc.n_cache].cpu().numpy()
        norms = np.linalg.norm(k_o, axis=2).T
        live = c_o > 0
        assert np.allclose(inv[live], 1.0 / norms[live], rtol=1e-5) and np.all(inv[~live] == -1.0)
    # the near-duplicate frames merged: the cache holds fewer entries than tokens seen
    assert tc.n_valid.max().item() < 3 * T


def test_merged_identical_keys_leave_attention_unchanged(cuda_ok):
    """Lemma 5.1 on the GPU: frame 2 repeats frame 1's keys (fresh values); merged with the log-size
    bias, the history branch equals attention over both frames unmerged."""
    import torch
    from kv_cache_compression_tma_b200 import ispa
    T, H, hd = 256, 2, 128
    k, v = frames(3, T, H, hd, seed=72)
    k[1] = k[0][np.argsort(inp.gaussian((T,), 72, 9))]             # the same keys in another order
    tc = ispa.TempCache(H, hd, capacity=2 * T)
    for f in range(2):
        tc.add_frame(dev(k[f], torch.bfloat16), dev(v[f], torch.bfloat16), 0.999)
    torch.cuda.synchronize()
    assert tc.n_valid.cpu().tolist() == [T] * H and int(tc.count[:, :T].sum()) == 2 * T * H
    kh, vh, bias = tc.segment()
    q = inp.round_bf16(inp.gaussian((200, H, hd), 72, 10).astype(np.float32) * np.float32(0.5))
    sink_k, sink_v = k[2][:64], v[2][:64]
    loc_k, loc_v = k[2][64:192], v[2][64:192]
    t = {n: dev(x, torch.bfloat16) for n, x in (("q", q), ("ks", sink_k), ("vs", sink_v), ("kl", loc_k), ("vl", loc_v))}
    out = ispa.dual_stream_attn(t["q"], t["ks"], t["vs"], t["kl"], t["vl"], kh, vh, kv_bias=(None, None, bias))
    torch.cuda.synchronize()
    hist_k = np.concatenate([k[0], k[1]])
    hist_v = np.concatenate([v[0], v[1]])
    ref = orc.dual_stream(q, sink_k, sink_v, loc_k, loc_v, hist_k, hist_v)
    assert rel(host(out["o_full"]), orc.stack_heads(ref["O_full"])) <= 1e-2
    assert rel(host(out["o_loc"]), orc.stack_heads(ref["O_loc"])) <= 1e-2
    assert np.max(np.abs(host(out["lse_hist"]) - ref["lse_hist"])) <= 2e-3
    assert rel(host(out["d"]), orc.stack_heads(ref["O_full"] - ref["O_loc"])) <= 1e-2


def test_biased_attention_against_oracle(cuda_ok):
    """A per-key bias on the history segment (ragged tiles, some -inf) against the oracle's biased
    softmax of the full key set."""
    import torch
    from kv_cache_compression_tma_b200 import ispa
    H, hd = 2, 128
    g = lambda shape, salt, sc=1.0: inp.round_bf16(inp.gaussian(shape, 73, salt, sc).astype(np.float32))
    q = g((150, H, hd), 1, 0.2)
    ks, vs = g((40, H, hd), 2), g((40, H, hd), 3)
    kl, vl = g((150, H, hd), 4), g((150, H, hd), 5)
    kh, vh = g((333, H, hd), 6), g((333, H, hd), 7)
    sizes = 1 + np.floor(np.abs(inp.gaussian((H, 336), 73, 8)) * 2.5).clip(0, 4)
    bias = np.log(sizes).astype(np.float32)
    bias[:, np.argsort(inp.gaussian((333,), 73, 9))[:40]] = -np.inf
    td = {n: dev(x, torch.bfloat16) for n, x in (("q", q), ("ks", ks), ("vs", vs), ("kl", kl), ("vl", vl),
                                                   ("kh", kh), ("vh", vh))}
    b = torch.from_numpy(bias).cuda()
    out = ispa.dual_stream_attn(td["q"], td["ks"], td["vs"], td["kl"], td["vl"], td["kh"], td["vh"],
                                kv_bias=(None, None, b[:, :333]))
    torch.cuda.synchronize()
    scale = 1.0 / math.sqrt(hd)
    for h in range(H):
        kf = np.concatenate([ks[:, h], kl[:, h], kh[:, h]])
        vf = np.concatenate([vs[:, h], vl[:, h], vh[:, h]])
        bf = np.concatenate([np.zeros(190), bias[h, :333]])
        o_ref, lse_ref = orc.biased_softmax_attention(q[:, h], kf, vf, bf, scale)
        got = host(out["o_full"]).reshape(150, H, hd)[:, h]
        assert rel(got, o_ref) <= 1e-2
        assert np.max(np.abs(np.logaddexp(host(out["lse_loc"])[h], host(out["lse_hist"])[h]) - lse_ref)) <= 2e-3
        o_loc_ref, _ = orc.softmax_attention(q[:, h], kf[:190], vf[:190], scale)
        assert rel(host(out["o_loc"]).reshape(150, H, hd)[:, h], o_loc_ref) <= 1e-2


def test_bias_on_cuda_cores_is_refused(cuda_ok):
    import torch
    from kv_cache_compression_tma_b200 import ispa
    x = torch.zeros((8, 1, 64), dtype=torch.bfloat16, device="cuda")
    b = torch.zeros((1, 8), dtype=torch.float32, device="cuda")
    with pytest.raises(ispa.IspaError) as e:
        ispa.dual_stream_attn(x, x, x, x, x, x, x, cuda_cores=True, kv_bias=(None, None, b))
    assert e.value.status == ispa.ISPA_ERR_UNSUPPORTED
