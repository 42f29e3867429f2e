"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Pivots must be identical (the oracle replays a GPU draw only inside the 1e-6
CDF window); outputs within 1e-5 (fp32 inputs) or 2e-3 (bf16 inputs) of the
oracle, as max |out - ref| / max |ref| per head.  Shapes span several tiles and
blocks per unit, with ragged tails."""

import numpy as np
import pytest
import torch

import oracle
from coreset_attention_approximation_b200 import wildcat
from coreset_attention_approximation_b200.workloads import WORKLOADS, make_inputs
from parity import TOL_OUT, compare, factor_shift, rel_err, run_gpu

pytestmark = pytest.mark.gpu


def test_tiny_fp32_full_workload():
    w = WORKLOADS["tiny"]
    rep = compare(*make_inputs(w), w.r, seed=0, tol_w=1e-5)
    assert rep["err_out"] <= 1e-5


def test_vit_full_workload():
    w = WORKLOADS["vit"]
    compare(*make_inputs(w), w.r, seed=0, tol_w=2e-3)


def test_diffusion_full_workload():
    w = WORKLOADS["diffusion"]
    compare(*make_inputs(w), w.r, seed=0, tol_w=2e-3)


def test_kv_reduced_gqa():
    w = WORKLOADS["kv"].replace(hq=8, hkv=2, n_k=8192, r=256)
    compare(*make_inputs(w), w.r, seed=3, tol_w=2e-3)


def test_kv_full_workload_two_units():
    """The KV-cache workload at full size (32 query heads over 8 kv heads,
    n = 32768, r = 1024, 256 queries) in the bench's launch configuration: the
    GPU runs all 8 units; the oracle checks every pivot, the factor, the weights
    and the outputs of the first and last unit (8 query heads)."""
    w = WORKLOADS["kv"]
    rep = compare(*make_inputs(w), w.r, seed=0, tol_w=2e-3, units=[0, w.hkv - 1])
    assert rep["err_out"] <= TOL_OUT[torch.bfloat16]


def test_long_reduced_many_blocks_per_unit():
    w = WORKLOADS["long"].replace(hq=1, hkv=1, n_k=16384, n_q=2048, r=512)
    compare(*make_inputs(w), w.r, seed=5, tol_w=2e-3)


@pytest.mark.parametrize("n,r,dtype", [(1000, 40, torch.float32), (777, 64, torch.bfloat16),
                                       (9, 5, torch.float32), (4099, 129, torch.bfloat16),
                                       (8, 8, torch.bfloat16)])
def test_ragged_sizes(n, r, dtype):
    w = WORKLOADS["vit"].replace(batch=2, hq=2, hkv=2, n_k=n, n_q=37, r=r, dtype="f32" if dtype == torch.float32
                                 else "bf16")
    compare(*make_inputs(w, seed=n), r, seed=n)


def test_r_equal_one():
    w = WORKLOADS["vit"].replace(batch=1, hq=2, hkv=2, n_k=300, n_q=50, r=1)
    compare(*make_inputs(w), 1, seed=2)


def test_rank_deficient_keys_stop_and_reproduce_exact_attention():
    g = torch.Generator().manual_seed(0)
    m, n, d, dv = 6, 640, 64, 64
    base = torch.randn(m, d, generator=g, dtype=torch.float64) * 0.25
    idx = torch.randint(0, m, (n,), generator=g)
    idx[:m] = torch.arange(m)
    K = base[idx][None, None].to(torch.float32).contiguous()
    V = torch.randn(1, 1, n, dv, generator=g).contiguous()
    Q = (torch.randn(1, 1, 33, d, generator=g) * 0.25).contiguous()
    res = run_gpu(Q, K, V, 32, seed=1)
    assert int(res["rank"][0, 0]) == m
    piv = res["piv"][0, 0].numpy()
    assert sorted(idx[piv[:m]].tolist()) == list(range(m)) and np.all(piv[m:] == -1)
    ex = oracle.exact_attention(Q[0, 0], K[0, 0], V[0, 0], 1.0 / np.sqrt(d))
    assert rel_err(res["out"][0, 0].numpy(), ex) <= 1e-4


def test_split_attention_with_empty_splits():
    """bf16 keys with 6 distinct rows and r = 512: the selection stops at rank
    6, so of the attention's four key splits (two query heads, one query tile
    each) only the first holds coreset rows; the combined rows are still exact
    attention."""
    g = torch.Generator().manual_seed(3)
    m, n, d, dv = 6, 1024, 64, 64
    base = torch.randn(m, d, generator=g, dtype=torch.float64) * 0.25
    idx = torch.randint(0, m, (n,), generator=g)
    idx[:m] = torch.arange(m)
    K = base[idx][None, None].to(torch.bfloat16).contiguous()
    V = torch.randn(1, 1, n, dv, generator=g, dtype=torch.float64).to(torch.bfloat16)
    Q = (torch.randn(1, 2, 33, d, generator=g, dtype=torch.float64) * 0.25).to(torch.bfloat16)
    res = run_gpu(Q, K, V, 512, seed=1)
    assert int(res["rank"][0, 0]) == m
    for h in range(2):
        ex = oracle.exact_attention(Q[0, h], K[0, 0], V[0, 0], 1.0 / np.sqrt(d))
        assert rel_err(res["out"][0, h].numpy(), ex) <= 2e-3


def test_all_keys_equal_gives_mean_of_values():
    n, d, dv = 256, 64, 64
    K = torch.full((1, 1, n, d), 0.05, dtype=torch.bfloat16)
    V = torch.randn(1, 1, n, dv, generator=torch.Generator().manual_seed(4)).to(torch.bfloat16)
    Q = torch.randn(1, 1, 16, d, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    res = run_gpu(Q, K, V, 8, seed=0)
    assert int(res["rank"][0, 0]) == 1
    mean = V[0, 0].double().mean(0).numpy()
    assert rel_err(res["out"][0, 0].numpy(), np.tile(mean, (16, 1))) <= 2e-3


def test_no_queries_runs_select_and_weights():
    w = WORKLOADS["vit"].replace(batch=1, hq=1, hkv=1, n_q=0)
    Q, K, V = make_inputs(w)
    res = run_gpu(Q, K, V, w.r, seed=0)
    o = oracle.forward(Q, K, V, w.r, seed=0, replay=(res["piv"].numpy(), res["rank"].numpy()))
    assert np.array_equal(res["piv"].numpy(), o["piv"])


def test_deterministic_bitwise():
    w = WORKLOADS["diffusion"].replace(batch=1, hq=2, hkv=2)
    Q, K, V = make_inputs(w)
    a = run_gpu(Q, K, V, w.r, seed=9)
    b = run_gpu(Q, K, V, w.r, seed=9)
    for k in ("piv", "rank", "F", "W", "out"):
        assert torch.equal(a[k], b[k]), k


def test_separate_calls_match_forward():
    w = WORKLOADS["kv"].replace(hq=4, hkv=2, n_k=2048, r=128, n_q=64)
    Q, K, V = [t.cuda() for t in make_inputs(w)]
    full = wildcat.forward(Q, K, V, w.r, seed=11)
    sel = wildcat.select(K, w.r, seed=11)
    wts = wildcat.weights(K, V, sel["piv"], sel["F"], sel["rank"], w.r)
    out = wildcat.attend(Q, wts["Ks"], wts["W"], sel["rank"], w.n_k)
    torch.cuda.synchronize()
    assert torch.equal(full["piv"], sel["piv"]) and torch.equal(full["F"], sel["F"])
    assert torch.equal(full["W"], wts["W"]) and torch.equal(full["out"], out)


def test_one_workspace_serves_the_three_calls():
    """The README's step-by-step use: a workspace sized for the whole problem
    is handed to select, weights and attend (attention with few queries, so
    the split attention's rows live in it too)."""
    w = WORKLOADS["kv"].replace(hq=8, hkv=2, n_k=4096, r=512, n_q=200)
    Q, K, V = [t.cuda() for t in make_inputs(w, seed=12)]
    full = wildcat.forward(Q, K, V, w.r, seed=12)
    ws = wildcat.workspace(wildcat.shape_of(Q, K, V, w.r), K.device)
    sel = wildcat.select(K, w.r, seed=12, ws=ws)
    wts = wildcat.weights(K, V, sel["piv"], sel["F"], sel["rank"], w.r, ws=ws, seed=12)
    out = wildcat.attend(Q, wts["Ks"], wts["W"], sel["rank"], w.n_k, ws=ws)
    assert wildcat.check_device_status(ws) == 0
    assert torch.equal(full["piv"], sel["piv"]) and torch.equal(full["W"], wts["W"]) and torch.equal(full["out"], out)


def test_wait_timeout_is_reported_and_context_survives():
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    assert wildcat.selftest_wait_timeout(ws, 200) == 0
    assert wildcat.check_device_status(ws) == 3          # WC_ERR_TIMEOUT
    assert wildcat.check_device_status(ws) == 0          # cleared
    w = WORKLOADS["tiny"]
    compare(*make_inputs(w), w.r, seed=0)


def test_full_long_workload_head0_and_properties():
    """The bench workload (long: 8 heads, n = 131072, r = 2048) in the bench's
    launch configuration.  Head 0 in full against the oracle: every pivot
    (replayed only inside the 1e-6 CDF window), the factor, the weights, and
    sampled outputs computed by the oracle from its own weights; on every head,
    properties that hold at any size."""
    w = WORKLOADS["long"]
    Q, K, V = make_inputs(w)
    res = run_gpu(Q, K, V, w.r, seed=0)
    piv, rank = res["piv"].numpy(), res["rank"].numpy()
    assert np.all(rank == w.r)
    beta = 1.0 / np.sqrt(w.d)
    K0 = K[0, 0].double().numpy()
    sel = oracle.rpcholesky(K0, w.r, beta, seed=0, unit=0, replay_piv=piv[0, 0], replay_rank=w.r)
    assert sel["failed_step"] == -1 and sel["rank"] == w.r, sel["fail_margin"]
    assert np.array_equal(sel["piv"], piv[0, 0])
    # the factor, 256 columns at a time (the library's F is the oracle's times exp(-M/2))
    scale = np.exp(-factor_shift(K0, beta) / 2)
    Fo = sel.pop("F")
    den = float(np.max(np.abs(Fo))) * scale
    worst = 0.0
    for c0 in range(0, w.r, 256):
        g = res["F"][0, 0, c0:c0 + 256, :w.n_k].double().numpy().T
        worst = max(worst, float(np.max(np.abs(g - Fo[:, c0:c0 + 256] * scale))))
    del Fo
    assert worst / den <= 1e-5
    Wo = oracle.nystrom_weights(K0, V[0, 0], piv[0, 0], w.r, beta)
    assert rel_err(res["W"][0, 0].numpy(), Wo) <= 2e-3
    rng = np.random.default_rng(0)
    qs = rng.choice(w.n_q, 256, replace=False)
    out_o = oracle.coreset_attend(Q[0, 0, qs], K0[piv[0, 0]], Wo, beta)
    assert rel_err(res["out"][0, 0, qs].numpy(), out_o) <= TOL_OUT[torch.bfloat16]
    F = res["F"]
    for h in range(w.hkv):
        p = piv[0, h]
        assert len(set(p.tolist())) == w.r
        L = F[0, h][:, p].numpy().T                              # L[a, c] = F[c, piv[a]]
        assert np.all(np.triu(L, 1) == 0.0) and np.all(np.diag(L) > 0.0)
        # F F^T reproduces the shifted kernel exp(beta K K^T - M) on sampled pivot rows
        Kh = K[0, h].double().numpy()
        M = factor_shift(Kh, beta)
        for a in rng.choice(w.r, 4, replace=False):
            i = rng.choice(w.n_k, 64, replace=False)
            Hrow = np.exp(beta * Kh[i] @ Kh[p[a]] - M)
            FFt = F[0, h][:, i].double().numpy().T @ L[a].astype(np.float64)
            assert rel_err(FFt, Hrow) <= 1e-4


def test_running_max_rescale_large_dynamic_range():
    """One key with a much larger norm than the rest is drawn first; in the
    weights GEMM its row meets its own (largest) logit only in a late key
    tile, so the running maximum grows by far more than the rescale
    threshold mid-row."""
    g = torch.Generator().manual_seed(7)
    n, d, dv, nq = 520, 64, 64, 200
    K = torch.randn(1, 1, n, d, generator=g) * 0.3
    # |k_500|^2 / sqrt(d) = 8 (11.5 in log2 units) against cross logits of about 1
    K[0, 0, 500] = 8.0 * torch.nn.functional.normalize(torch.randn(d, generator=g), dim=0)
    V = torch.randn(1, 1, n, dv, generator=g)
    Q = torch.randn(1, 1, nq, d, generator=g) * 0.3
    Q[0, 0, :20] = 0.5 * K[0, 0, 500]
    Q, K, V = Q.to(torch.bfloat16), K.to(torch.bfloat16), V.to(torch.bfloat16)
    compare(Q, K, V, 48, seed=1)
    res = run_gpu(Q, K, V, 48, seed=1)
    assert int(res["piv"][0, 0, 0]) == 500 and int(res["rank"][0, 0]) == 48


@pytest.mark.parametrize("d,dv", [(32, 96), (128, 64), (64, 128), (256, 256), (8, 8), (256, 8)])
def test_other_head_widths_bf16(d, dv):
    # (128, 64) and (64, 128) run on the tensor-core kernel, the others on CUDA cores;
    # 8 and 256 are the narrowest and widest heads the library takes
    w = WORKLOADS["vit"].replace(batch=1, hq=4, hkv=2, n_k=1500, n_q=300, d=d, dv=dv, r=100)
    compare(*make_inputs(w, seed=d + dv), w.r, seed=3)


@pytest.mark.parametrize("d,dv", [(256, 256), (8, 8)])
def test_extreme_head_widths_fp32(d, dv):
    w = WORKLOADS["tiny"].replace(batch=1, hq=2, hkv=2, n_k=700, n_q=90, d=d, dv=dv, r=40)
    rep = compare(*make_inputs(w, seed=d + 7), w.r, seed=5, tol_w=1e-5)
    assert rep["err_out"] <= 1e-5


def test_large_key_norms_factor_stays_finite():
    """Keys with beta |k|^2 around 300 (norms near 50 at d = 64): the unshifted
    factor would reach exp(150) and overflow fp32; the selection works on the
    kernel shifted by M = max beta |k_i|^2, so F stays finite and the pivots,
    weights and outputs match the oracle's (fp64, unshifted)."""
    w = WORKLOADS["vit"].replace(batch=1, hq=2, hkv=2, n_k=512, n_q=64, r=32)
    Q, K, V = make_inputs(w, seed=21)
    g = torch.Generator().manual_seed(21)
    scale = 50.0 / K.double().norm(dim=-1, keepdim=True).clamp_min(1e-3)
    K = (K.double() * scale * (0.8 + 0.2 * torch.rand(K.shape[:-1] + (1,), generator=g, dtype=torch.float64))).to(K.dtype)
    Q = (Q.double() * 0.02).to(Q.dtype)
    rep = compare(Q, K, V, w.r, seed=21, tol_w=2e-3)
    res = run_gpu(Q, K, V, w.r, seed=21)
    assert torch.isfinite(res["F"]).all() and res["F"].abs().max() <= 1.0 + 1e-6, rep


@pytest.mark.parametrize("bins", [1, 4])
def test_host_pipeline_matches_forward(bins):
    """Three different host batches through the double-buffered host pipeline
    give, bit for bit, the outputs of separate forward calls (same seed)."""
    w = WORKLOADS["diffusion"].replace(batch=1, hq=4, hkv=2, n_k=4096, n_q=1000, r=256)
    batches = [make_inputs(w, seed=s) for s in (11, 12, 13)]
    pinned = [tuple(t.pin_memory() for t in b) for b in batches]
    outs = [torch.empty(w.batch, w.hq, w.n_q, w.dv, dtype=torch.float32).pin_memory() for _ in batches]
    pipe = wildcat.HostPipeline(*pinned[0], w.r, seed=4, bins=bins)
    pipe.run([(q, k, v, o) for (q, k, v), o in zip(pinned, outs)])
    assert pipe.wait() == 0
    for (Q, K, V), o in zip(batches, outs):
        ref = run_gpu(Q, K, V, w.r, seed=4, bins=bins)["out"]
        assert torch.equal(o, ref)
    # a second run on the same pipeline (buffers and events reused)
    pipe.run([(*pinned[2], outs[0])])
    assert pipe.wait() == 0
    assert torch.equal(outs[0], outs[2])


def test_maximum_coreset_size():
    """r = 4096, the largest coreset the library takes, on keys whose kernel
    stays full rank (unit directions at norm 6, d = 64: diagonally dominant),
    so every one of the 4096 steps runs; 6000 keys leave unchosen mass, as in
    any real use."""
    w = WORKLOADS["vit"].replace(batch=1, hq=2, hkv=1, n_k=6000, n_q=200, r=4096)
    Q, K, V = make_inputs(w, seed=41)
    g = torch.Generator().manual_seed(41)
    K = (torch.nn.functional.normalize(torch.randn(K.shape, generator=g, dtype=torch.float64), dim=-1) * 6.0).to(K.dtype)
    compare(Q, K, V, w.r, seed=41, tol_w=2e-3)
    assert int(run_gpu(Q, K, V, w.r, seed=41)["rank"][0, 0]) == w.r


def test_many_keys_in_one_unit():
    """3,000,037 keys in one unit (293 co-resident blocks of 10240 rows, a
    ragged last block), the whole path against the oracle."""
    w = WORKLOADS["vit"].replace(batch=1, hq=2, hkv=1, n_k=3_000_037, n_q=300, r=16)
    compare(*make_inputs(w, seed=43), w.r, seed=43, tol_w=2e-3)


def test_keys_beyond_the_coresident_limit_are_refused():
    """The select keeps a unit's residual diagonal in the shared memory of
    co-resident blocks; beyond what the GPU holds at once (about 3.6 million
    keys a unit on 148 SMs) it returns WC_ERR_UNSUPPORTED without launching."""
    w = WORKLOADS["vit"].replace(batch=1, hq=1, hkv=1, n_k=4_194_341, n_q=0, r=4)
    dev = torch.device("cuda")
    K = torch.zeros(1, 1, w.n_k, w.d, dtype=torch.bfloat16, device=dev)
    with pytest.raises(wildcat.WildcatError) as e:
        wildcat.select(K, w.r, seed=0)
    assert e.value.code == 4
    torch.cuda.synchronize()


@pytest.mark.parametrize("kw", [{}, {"bins": 4}, {"bins": 2, "center": True}])
def test_forward_graph_replays_match_eager(kw):
    """The forward pass captured into a CUDA graph (cooperative select launch
    included: 16384 keys a unit run on several blocks) and replayed on new
    inputs copied in place gives, bit for bit, the eager pass's results."""
    w = WORKLOADS["long"].replace(hq=4, hkv=2, n_k=16384, n_q=1000, r=256)
    inputs = [make_inputs(w, seed=s) for s in (21, 22)]
    dev = torch.device("cuda")
    Q, K, V = [t.to(dev) for t in inputs[0]]
    g = wildcat.ForwardGraph(Q, K, V, w.r, seed=3, **kw)
    for Qh, Kh, Vh in inputs:
        Q.copy_(Qh)
        K.copy_(Kh)
        V.copy_(Vh)
        o = g.replay()
        torch.cuda.synchronize()
        assert wildcat.check_device_status(g.ws) == 0
        ref = run_gpu(Qh, Kh, Vh, w.r, seed=3, **kw)
        for k in ("out", "piv", "rank", "F", "W"):
            assert torch.equal(o[k].cpu(), ref[k]), k


@pytest.mark.parametrize("d,deficient", [(128, False), (64, False), (128, True)])
def test_attention_many_query_tiles(d, deficient):
    """Attention over 40 ragged query tiles x 8 heads (no key split); r = 640
    gives an odd number of key tiles (5); with `deficient` the second kv head's
    keys have 6 distinct rows, so its query tiles see one key tile while the
    first head's see five."""
    w = WORKLOADS["long"].replace(hq=8, hkv=2, n_k=4096, n_q=5000, r=640, d=d)
    Q, K, V = make_inputs(w, seed=51)
    if deficient:
        g = torch.Generator().manual_seed(51)
        base = torch.randn(6, d, generator=g, dtype=torch.float64) * 0.3
        idx = torch.randint(0, 6, (w.n_k,), generator=g)
        idx[:6] = torch.arange(6)
        K[0, 1] = base[idx].to(K.dtype)
    rep = compare(Q, K, V, w.r, seed=51, tol_w=2e-3)
    if deficient:
        res = run_gpu(Q, K, V, w.r, seed=51)
        assert int(res["rank"][0, 1]) == 6 and int(res["rank"][0, 0]) == w.r, rep
