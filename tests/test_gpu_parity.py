"""Parity of the CUDA path (through the C ABI) against the fp64 oracle.

Routing: top-k indices and per-expert counts bit-exact against the oracle's
top-k applied to the device's own fp32 logits; logits within 1e-4 of the
fp64 scores (row-scaled).  Layer outputs: bf16 layers within max-abs 2e-2 and
relative L2 1e-2 of fp64; fp32 layers within 1e-4 (relative).  Dispatch
(histogram, scan, permutation) is integer work and is compared exactly.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_mixture_experts_10_b200 as moe
from moe_inputs import ACT_GELU, ACT_SWIGLU, WORKLOADS, Workload, make_inputs
from sparse_mixture_experts_10_b200 import build as moe_build
from tests import parity_helpers as ph

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    moe_build.build()
    moe.load_library()
    assert moe.moe_get_device_status() == 0
    yield
    torch.cuda.empty_cache()


class Layer:
    """Config, weights and workspace of one workload on the device."""

    def __init__(self, wl: Workload, inp):
        self.wl, self.inp = wl, inp
        self.cfg = moe.make_config(wl.D, wl.H, wl.N, wl.K, wl.act, moe.dtype_code(wl.dtype), wl.has_bias,
                                   wl.n_shared, wl.capacity_factor, wl.overflow)
        self.w = moe.make_weights(inp["W_g"], inp["W1"], inp["W2"], inp["b_g"], inp["b1"], inp["b2"],
                                  inp.get("b_sel"), inp.get("S1"), inp.get("sb1"), inp.get("S2"), inp.get("sb2"))

    def forward(self, x=None, y_dtype=torch.float32, with_aux=True):
        x = self.inp["x"] if x is None else x
        T, N = x.shape[0], self.wl.N
        ws = moe.alloc_workspace(self.cfg, max(T, 1))
        y = torch.full((T, self.wl.D), float("nan"), dtype=y_dtype, device="cuda")
        aux = None
        if with_aux:
            aux = dict(counts=torch.full((N,), -1, dtype=torch.int32, device="cuda"),
                       importance=torch.full((N,), -1.0, device="cuda"),
                       p_mean=torch.full((N,), -1.0, device="cuda"),
                       scalars=torch.full((4,), -1.0, device="cuda"))
        caux = moe.make_aux(**aux) if aux else None
        moe.check(moe.moe_forward(self.cfg, x, T, self.w, y, moe.dtype_code(y_dtype), caux, ws, ws.numel()),
                  "moe_forward")
        torch.cuda.synchronize()
        assert moe.moe_get_device_status() == 0
        return y, ws, aux

    def views(self, ws, T):
        """The routing results and dispatch maps moe_forward left in the workspace."""
        L = moe.moe_get_workspace_layout(self.cfg, T)
        N, K = self.wl.N, self.wl.K

        def v(off, n, dt):
            return ws[off:off + n * torch.tensor([], dtype=dt).element_size()].view(dt)

        es_dt = self.wl.dtype
        return dict(
            logits=v(L.logits, T * N, torch.float32).view(T, N).cpu().numpy(),
            idx=v(L.topk_idx, T * K, torch.int32).view(T, K).cpu().numpy(),
            w=v(L.topk_w, T * K, torch.float32).view(T, K).cpu().numpy(),
            counts=v(L.counts, N, torch.int32).cpu().numpy(),
            offsets=v(L.offsets, N + 1, torch.int32).cpu().numpy(),
            row_offsets=v(L.row_offsets, N + 1, torch.int32).cpu().numpy(),
            perm_slot=v(L.perm_slot, L.rows_cap, torch.int32).cpu().numpy(),
            slot_row=v(L.slot_row, T * K, torch.int32).cpu().numpy(),
            x_perm=v(L.x_perm, L.rows_cap * self.wl.D, es_dt).view(L.rows_cap, self.wl.D),
            rows_cap=L.rows_cap,
        )


def check_routing(V, ref_scores, K, inp, C=None):
    """Logits within tolerance, top-k bit-exact on the device's logits (plus any selection bias,
    added in fp32 as the device does), counts exact (the accepted ones under a capacity C)."""
    ph.assert_logits_close(V["logits"], ref_scores)
    sel = oracle.select_topk(ph.selection_scores(V["logits"], inp).astype(np.float64), K)
    np.testing.assert_array_equal(V["idx"], sel)
    N = V["counts"].shape[0]
    counts = np.bincount(sel.ravel(), minlength=N)
    np.testing.assert_array_equal(V["counts"], counts if C is None else np.minimum(counts, C))


def check_dispatch(V, x, K, C=None):
    """The permutation is the stable counting sort of the (token, slot) pairs by expert; with a
    capacity C each expert's segment holds its first C pairs (the oracle's drop decision) and
    the dropped pairs have no row."""
    idx = V["idx"]
    T = idx.shape[0]
    N = V["counts"].shape[0]
    flat = idx.ravel()
    keep = np.ones(T * K, dtype=bool) if C is None else oracle.capacity_keep(idx, N, C).ravel().astype(bool)
    counts = np.bincount(flat[keep], minlength=N)
    np.testing.assert_array_equal(V["counts"], counts)
    np.testing.assert_array_equal(V["offsets"], np.concatenate([[0], np.cumsum(counts)]))
    padded = (counts + 127) // 128 * 128
    np.testing.assert_array_equal(V["row_offsets"], np.concatenate([[0], np.cumsum(padded)]))
    ro = V["row_offsets"]
    for e in range(N):
        seg = V["perm_slot"][ro[e]:ro[e + 1]]
        expect = np.nonzero((flat == e) & keep)[0]
        np.testing.assert_array_equal(seg[:counts[e]], expect)
        assert np.all(seg[counts[e]:] == -1)
        np.testing.assert_array_equal(V["slot_row"][expect], np.arange(ro[e], ro[e] + counts[e]))
    assert np.all(V["slot_row"][~keep] == -1)
    kept = np.nonzero(keep)[0]
    rows = V["slot_row"][kept]
    tok = kept // K
    xp = V["x_perm"][torch.from_numpy(rows.astype(np.int64)).cuda()]
    assert torch.equal(xp, x[torch.from_numpy(tok).cuda()])


def run_full(wl, inp, y_dtype=torch.float32):
    layer = Layer(wl, inp)
    T = inp["x"].shape[0]
    y, ws, aux = layer.forward(y_dtype=y_dtype)
    V = layer.views(ws, T)
    ref = ph.oracle_full_layer(inp, wl, wl.K, gpu_logits=V["logits"])
    check_routing(V, ref["scores"], wl.K, inp, ref.get("capacity"))
    ph.assert_weights_close(V["w"], ref["w"], ref["scores"])
    check_dispatch(V, inp["x"], wl.K, ref.get("capacity"))
    errs = ph.assert_y_close(y.float().cpu().numpy(), ref["y"], wl.dtype if y_dtype == torch.float32 else y_dtype)
    return layer, y, ws, aux, V, ref, errs


def check_aux(aux, V, N, K):
    st = oracle.aux_stats(V["logits"].astype(np.float64), V["idx"], V["w"].astype(np.float64), N)
    np.testing.assert_array_equal(aux["counts"].cpu().numpy(), st["counts"].astype(np.int32))
    np.testing.assert_allclose(aux["importance"].cpu().numpy(), st["importance"], rtol=1e-5, atol=1e-5)
    np.testing.assert_allclose(aux["p_mean"].cpu().numpy(), st["p_mean"], rtol=1e-5, atol=1e-7)
    sc = aux["scalars"].cpu().numpy()
    np.testing.assert_allclose(sc, [st["switch"], st["simple"], st["cv2_importance"], st["cv2_load"]],
                               rtol=1e-4, atol=1e-6)


# ----------------------------------------------------------------------------- tiny fp32
def test_tiny_fp32_full_layer():
    wl = WORKLOADS["tiny"]
    inp = make_inputs(wl, "cuda")
    layer, y, ws, aux, V, ref, errs = run_full(wl, inp)
    check_aux(aux, V, wl.N, wl.K)


def test_tiny_fp32_random_biases_and_router_bias():
    wl = WORKLOADS["tiny"].with_(random_bias=True, zipf_s=0.5)
    inp = make_inputs(wl, "cuda", T=300)
    run_full(wl, inp)


@pytest.mark.parametrize("T", [1, 2, 33, 127, 129])
def test_tiny_fp32_small_and_ragged_batches(T):
    wl = WORKLOADS["tiny"].with_(random_bias=True)
    inp = make_inputs(wl, "cuda", T=T)
    run_full(wl, inp)


def test_topk_equals_n_and_top1():
    for N, K in [(8, 8), (8, 1), (6, 6), (32, 3), (20, 5)]:
        wl = WORKLOADS["tiny"].with_(N=N, K=K, random_bias=True)
        inp = make_inputs(wl, "cuda", T=200)
        run_full(wl, inp)


def test_single_expert_top1():
    wl = WORKLOADS["tiny"].with_(N=1, K=1, random_bias=True)
    inp = make_inputs(wl, "cuda", T=100)
    layer, y, ws, aux, V, ref, errs = run_full(wl, inp)
    assert np.all(V["w"] == 1.0)


def test_all_tokens_on_one_expert_and_empty_experts():
    wl = WORKLOADS["tiny"].with_(random_bias=True)
    inp = make_inputs(wl, "cuda", T=400)
    inp["b_g"] = torch.zeros(wl.N, device="cuda")
    inp["b_g"][5] = 100.0
    inp["b_g"][2] = 50.0
    layer, y, ws, aux, V, ref, errs = run_full(wl, inp)
    assert np.all(V["idx"][:, 0] == 5) and np.all(V["idx"][:, 1] == 2)
    assert V["counts"][5] == 400 and V["counts"].sum() == 800
    check_aux(aux, V, wl.N, wl.K)


def test_exact_ties_go_to_lower_index():
    wl = WORKLOADS["tiny"].with_(random_bias=True)
    inp = make_inputs(wl, "cuda", T=256)
    Wg = inp["W_g"]
    Wg[:, 6] = Wg[:, 1]
    Wg[:, 3] = Wg[:, 1]
    layer, y, ws, aux, V, ref, errs = run_full(wl, inp)
    for t in range(256):
        tied = [e for e in V["idx"][t].tolist() if e in (1, 3, 6)]
        assert tied == sorted(tied)
        if 3 in tied:
            assert 1 in tied
        if 6 in tied:
            assert 1 in tied and 3 in tied


def test_zero_tokens():
    wl = WORKLOADS["tiny"]
    inp = make_inputs(wl, "cuda", T=4)
    layer = Layer(wl, inp)
    ws = moe.alloc_workspace(layer.cfg, 1)
    aux = dict(counts=torch.full((wl.N,), 7, dtype=torch.int32, device="cuda"),
               importance=torch.ones(wl.N, device="cuda"), p_mean=torch.ones(wl.N, device="cuda"),
               scalars=torch.ones(4, device="cuda"))
    y = torch.empty(0, wl.D, device="cuda")
    moe.check(moe.moe_forward(layer.cfg, inp["x"], 0, layer.w, y, moe.MOE_F32, moe.make_aux(**aux), ws, ws.numel()))
    torch.cuda.synchronize()
    for k in aux:
        assert torch.all(aux[k] == 0), k
    cnt = torch.full((wl.N,), 3, dtype=torch.int32, device="cuda")
    moe.check(moe.moe_route(layer.cfg, inp["x"], 0, layer.w, None, None, None, cnt, ws, ws.numel()))
    torch.cuda.synchronize()
    assert torch.all(cnt == 0)


@pytest.mark.parametrize("N,K,T", [(8, 2, 2500), (16, 3, 2100), (32, 4, 2049), (6, 2, 2080)])
def test_chunked_router_path(N, K, T):
    """T >= 2048 with N <= 32 takes the chunked router (W_g staged in shared memory)."""
    wl = WORKLOADS["tiny"].with_(N=N, K=K, random_bias=True, zipf_s=0.3)
    inp = make_inputs(wl, "cuda", T=T)
    run_full(wl, inp)


@pytest.mark.parametrize("dtype,N,K", [(torch.float32, 40, 3), (torch.float32, 64, 6), (torch.bfloat16, 64, 4),
                                       (torch.bfloat16, 300, 8), (torch.bfloat16, 40, 2), (torch.bfloat16, 64, 1)])
def test_gemm_router_path(dtype, N, K):
    """N > 32 takes the router GEMM (SIMT for fp32, tcgen05 dense tile for bf16) and the top-k kernel.
    bf16 with K <= 2: the combine folds into the down projection and the permute kernel clears y."""
    wl = Workload("many_experts", 11, 700, 256, 128, N, K, ACT_SWIGLU if dtype == torch.bfloat16 else ACT_GELU,
                  dtype, dtype == torch.float32, 0.05, zipf_s=0.5, random_bias=True)
    inp = make_inputs(wl, "cuda")
    layer, y, ws, aux, V, ref, errs = run_full(wl, inp)
    check_aux(aux, V, wl.N, wl.K)


# ----------------------------------------------------------------------------- bf16, tensor cores
def test_gpt2_bf16_reduced_batch_full_layer():
    wl = WORKLOADS["gpt2"]
    inp = make_inputs(wl, "cuda", T=1000)
    layer, y, ws, aux, V, ref, errs = run_full(wl, inp)
    check_aux(aux, V, wl.N, wl.K)


def test_gpt2_bf16_random_biases():
    wl = WORKLOADS["gpt2"].with_(random_bias=True)
    inp = make_inputs(wl, "cuda", T=777)
    run_full(wl, inp)


def test_bf16_ragged_dims_gelu_and_swiglu():
    """D and H not multiples of the 64-wide K slice or of the 256/128-wide column tiles."""
    for act in (ACT_GELU, ACT_SWIGLU):
        wl = Workload("ragged", 9, 300, 200, 328, 5, 2, act, torch.bfloat16, act == ACT_GELU, 0.05,
                      random_bias=True)
        inp = make_inputs(wl, "cuda")
        run_full(wl, inp)


@pytest.mark.parametrize("act,T,seed", [(ACT_SWIGLU, 1500, 0), (ACT_GELU, 1300, 1), (ACT_SWIGLU, 1100, 2)])
def test_bf16_pair_tiles_with_ragged_segments(act, T, seed):
    """Enough rows for the 2-CTA (256-row) tiles; skewed routing leaves experts with odd numbers of
    128-row tiles, so some pair tiles have their upper half past the expert's segment."""
    wl = Workload("pairs", 12 + seed, T, 512, 1024, 8, 2, act, torch.bfloat16, act == ACT_GELU, 0.04,
                  zipf_s=0.7, random_bias=True)
    inp = make_inputs(wl, "cuda")
    layer, y, ws, aux, V, ref, errs = run_full(wl, inp)
    counts = V["counts"]
    assert any(((c + 127) // 128) % 2 == 1 for c in counts if c > 0)


@pytest.mark.parametrize("act", [ACT_GELU, ACT_SWIGLU])
def test_hidden_activations_match_oracle(act):
    """The up-projection epilogue (GELU with bias, or SwiGLU) element by element: every hidden value of
    sampled permuted rows is within bf16 rounding of the oracle's fp64 hidden layer."""
    wl = Workload("hidden", 20 + act, 1200, 256, 384, 4, 2, act, torch.bfloat16, act == ACT_GELU, 0.08,
                  random_bias=True)
    inp = make_inputs(wl, "cuda")
    layer = Layer(wl, inp)
    y, ws, aux = layer.forward()
    V = layer.views(ws, wl.T)
    L = moe.moe_get_workspace_layout(layer.cfg, wl.T)
    h = ws[L.h:L.h + L.rows_cap * wl.H * 2].view(torch.bfloat16).view(L.rows_cap, wl.H).float().cpu().numpy()
    rng = np.random.default_rng(5)
    slots = rng.choice(wl.T * wl.K, size=40, replace=False)
    xb = ph.host(inp["x"])
    for f in slots:
        t, j = divmod(int(f), wl.K)
        e = int(V["idx"][t, j])
        row = int(V["slot_row"][f])
        xr = oracle.load_rows(xb, oracle.BF16, [t])[0]
        b1 = None if inp["b1"] is None else ph.host(inp["b1"][e])
        b2 = None if inp["b2"] is None else ph.host(inp["b2"][e])
        _, hid = oracle.expert(xr, act, oracle.BF16, ph.host(inp["W1"][e]), ph.host(inp["W2"][e]), b1, b2,
                               return_hidden=True)
        # bf16 keeps 8 significant bits: half an ulp is 2^-9 of the value; plus fp32 accumulation noise
        np.testing.assert_allclose(h[row], hid, rtol=2.0 ** -8, atol=1e-4)


def test_bf16_output_dtype():
    wl = WORKLOADS["gpt2"]
    inp = make_inputs(wl, "cuda", T=300)
    layer = Layer(wl, inp)
    y32, ws, _ = layer.forward(y_dtype=torch.float32, with_aux=False)
    y16, _, _ = layer.forward(y_dtype=torch.bfloat16, with_aux=False)
    assert torch.equal(y16, y32.to(torch.bfloat16))


def test_gpt2_full_size_sampled_rows():
    wl = WORKLOADS["gpt2"]
    inp = make_inputs(wl, "cuda")
    layer = Layer(wl, inp)
    y, ws, aux = layer.forward()
    V = layer.views(ws, wl.T)
    sel = oracle.select_topk(ph.selection_scores(V["logits"], inp).astype(np.float64), wl.K)
    np.testing.assert_array_equal(V["idx"], sel)
    check_dispatch(V, inp["x"], wl.K)
    check_aux(aux, V, wl.N, wl.K)
    rows = ph.sample_rows(wl.T, 48, V["idx"], wl.N, seed=2)
    ref = ph.oracle_rows(inp, wl, wl.K, rows, V["logits"])
    ph.assert_logits_close(V["logits"][rows], ref["scores"])
    ph.assert_weights_close(V["w"][rows], ref["w"], ref["scores"])
    ph.assert_y_close(y[torch.from_numpy(rows).cuda()].cpu().numpy(), ref["y"], wl.dtype)


def _full_size_sampled(name, n_rows, seed, every_expert=False):
    wl = WORKLOADS[name]
    inp = make_inputs(wl, "cuda")
    layer = Layer(wl, inp)
    y, ws, aux = layer.forward()
    V = layer.views(ws, wl.T)
    sel = oracle.select_topk(ph.selection_scores(V["logits"], inp).astype(np.float64), wl.K)
    np.testing.assert_array_equal(V["idx"], sel)
    np.testing.assert_array_equal(V["counts"], np.bincount(sel.ravel(), minlength=wl.N))
    check_aux(aux, V, wl.N, wl.K)
    rows = ph.sample_rows(wl.T, n_rows, V["idx"], wl.N, seed=seed, least_loaded=2)
    if every_expert:
        # the first and the last token routed to every live expert: their rows open and close
        # the expert's segment, so every expert's first tile and ragged last tile are compared
        ends = ph.expert_end_rows(V["idx"], wl.N)
        rows = np.union1d(rows, ends)
        live = np.nonzero(V["counts"] > 0)[0]
        covered = np.unique(V["idx"][rows])
        assert np.array_equal(covered, live), "a live expert has no compared output row"
        # logits of a strided subset of 1024 rows against the oracle's fp64 scores
        strided = np.arange(0, wl.T, max(1, wl.T // 1024))[:1024]
        ph.assert_logits_close(V["logits"][strided], ph.oracle_scores(inp, wl, strided))
    ref = ph.oracle_rows(inp, wl, wl.K, rows, V["logits"])
    ph.assert_logits_close(V["logits"][rows], ref["scores"])
    ph.assert_weights_close(V["w"][rows], ref["w"], ref["scores"])
    errs = ph.assert_y_close(y[torch.from_numpy(rows).cuda()].cpu().numpy(), ref["y"], wl.dtype)
    del inp, layer, ws, y
    torch.cuda.empty_cache()
    return errs


def test_mixtral_full_size_sampled_rows():
    _full_size_sampled("mixtral", 24, 3)


@pytest.mark.parametrize("name", ["deepseek", "deepseek_zipf", "deepseek_shared"])
def test_deepseek_full_size_sampled_rows(name):
    _full_size_sampled(name, 12, 4, every_expert=True)


@pytest.mark.parametrize("name", ["decode1", "decode8", "decode64"])
def test_decode_full_layer(name):
    wl = WORKLOADS[name]
    inp = make_inputs(wl, "cuda")
    run_full(wl, inp)


@pytest.mark.parametrize("name,wl", [
    ("gpt-oss T=1", WORKLOADS["decode1"]),
    ("gpt-oss T=8 skewed, bias, capacity", WORKLOADS["decode8"].with_(zipf_s=1.5, sel_s=0.5, capacity_factor=1.0)),
    ("gpt-oss T=64", WORKLOADS["decode64"]),
    ("GELU + biases, N=6, T=37", Workload("fused_gelu", 70, 37, 1024, 1024, 6, 2, ACT_GELU, torch.bfloat16, True, 0.03,
                                         random_bias=True, zipf_s=0.3)),
    ("ragged D/H, T=5", Workload("fused_rag", 71, 5, 1000, 712, 12, 3, ACT_SWIGLU, torch.bfloat16, False, 0.04,
                                 zipf_s=0.5)),
], ids=lambda v: v if isinstance(v, str) else "")
def test_decode_layer_is_one_kernel(name, wl):
    """Few tokens: routing, dispatch, both expert GEMMs and the combine run as one cooperative
    kernel after the counter clear (two launches per layer call), with the same results as the
    oracle (routing bit-exact, y within the bf16 tolerance, statistics)."""
    inp = make_inputs(wl, "cuda")
    layer = Layer(wl, inp)
    layer.forward(with_aux=False)            # the device's attributes are set up once
    n0 = moe.moe_launch_count()
    layer.forward(with_aux=False)
    assert moe.moe_launch_count() - n0 == 2
    run_layer, y, ws, aux, V, ref, errs = run_full(wl, inp)
    check_aux(aux, V, wl.N, wl.K)


@pytest.mark.parametrize("name,wl", [
    ("gpt-oss T=2", WORKLOADS["decode1"].with_(T=2)),
    ("gpt-oss T=2 skewed, capacity drop", WORKLOADS["decode1"].with_(T=2, zipf_s=2.0, capacity_factor=0.5)),
    ("GELU + biases, T=4 K=2", Workload("small_gelu", 72, 4, 1024, 1024, 6, 2, ACT_GELU, torch.bfloat16, True,
                                        0.03, random_bias=True, zipf_s=0.3)),
    ("ragged D/H, T=2 K=3, selection bias", Workload("small_rag", 73, 2, 1000, 712, 12, 3, ACT_SWIGLU,
                                                     torch.bfloat16, False, 0.04, zipf_s=0.5, sel_s=0.5)),
    ("one token, K=8 of 32", Workload("small_k8", 74, 1, 512, 384, 32, 8, ACT_SWIGLU, torch.bfloat16, False, 0.05)),
], ids=lambda v: v if isinstance(v, str) else "")
def test_decode_few_tokens(name, wl):
    """One to four tokens: the one-kernel decode path (two launches per layer call, counter clear
    included) with routing bit-exact, y within the bf16 tolerance and the statistics, for dropped
    slots, ragged D / H, a selection bias and K = 8."""
    inp = make_inputs(wl, "cuda")
    layer = Layer(wl, inp)
    layer.forward(with_aux=False)
    n0 = moe.moe_launch_count()
    layer.forward(with_aux=False)
    assert moe.moe_launch_count() - n0 == 2
    run_layer, y, ws, aux, V, ref, errs = run_full(wl, inp)
    check_aux(aux, V, wl.N, wl.K)


@pytest.mark.parametrize("N,K,T", [(12, 3, 300), (32, 4, 300), (6, 2, 1), (20, 4, 40), (32, 8, 64), (33, 2, 50)])
def test_bf16_router_paths(N, K, T):
    """bf16 routers: the SIMT router with 16 and 32 padded experts (T > 64), the few-token
    router at several sizes (T <= 64, N <= 32) and the tensor-core router below decode size."""
    wl = Workload("routers", 20 + N, T, 256, 128, N, K, ACT_SWIGLU, torch.bfloat16, False, 0.05,
                  zipf_s=0.4, random_bias=True)
    inp = make_inputs(wl, "cuda")
    layer, y, ws, aux, V, ref, errs = run_full(wl, inp)
    check_aux(aux, V, wl.N, wl.K)


@pytest.mark.parametrize("T", [1, 20, 50])
def test_bf16_decode_gelu_with_bias(T):
    """Decode path with the GELU expert and its biases; tile counts small enough for stream-K
    (cut tiles summed in piece order) with 16, 32 and 64 token columns."""
    wl = Workload("decode_gelu", 30, T, 1024, 1024, 6, 2, ACT_GELU, torch.bfloat16, True, 0.03,
                  random_bias=True)
    inp = make_inputs(wl, "cuda")
    run_full(wl, inp)


@pytest.mark.parametrize("K", [1, 3])
def test_bf16_prefill_k1_and_k3(K):
    """Top-1 (combine folded into the down projection) and top-3 (z in permuted row order,
    combined by gathering each token's rows in slot order)."""
    wl = Workload("prefill_k", 31 + K, 700, 512, 512, 6, K, ACT_SWIGLU, torch.bfloat16, False, 0.04,
                  zipf_s=0.5, random_bias=True)
    inp = make_inputs(wl, "cuda")
    run_full(wl, inp)


# ----------------------------------------------------------------------------- shared expert, selection bias
SHARED_CASES = [
    # (name, workload, T): every router and GEMM family with a shared expert and a selection bias
    ("fp32_gelu_bias", Workload("sh_f32", 50, 300, 64, 256, 8, 2, ACT_GELU, torch.float32, True, 0.05,
                                zipf_s=0.6, random_bias=True, n_shared=1, sel_s=0.6), None),
    ("fp32_swiglu_n40", Workload("sh_f32b", 51, 200, 64, 128, 40, 3, ACT_SWIGLU, torch.float32, False, 0.05,
                                 zipf_s=0.4, n_shared=1, sel_s=0.8), None),
    ("bf16_gelu_simt_router_k2", Workload("sh_gelu", 52, 1100, 256, 512, 6, 2, ACT_GELU, torch.bfloat16, True,
                                          0.04, zipf_s=0.7, random_bias=True, n_shared=1, sel_s=0.7), None),
    ("bf16_swiglu_tc_router", Workload("sh_tc", 53, 900, 256, 256, 64, 4, ACT_SWIGLU, torch.bfloat16, False,
                                       0.05, zipf_s=0.5, n_shared=1, sel_s=0.5), None),
    ("bf16_pairs_ragged", Workload("sh_pairs", 54, 1500, 512, 1024, 8, 2, ACT_SWIGLU, torch.bfloat16, False, 0.04,
                                   zipf_s=0.7, n_shared=1, sel_s=0.35), None),
    ("decode1", WORKLOADS["decode1"].with_(n_shared=1, sel_s=0.5, zipf_s=0.5), None),
    ("decode8", WORKLOADS["decode8"].with_(n_shared=1, sel_s=0.5, zipf_s=0.5), None),
    ("decode_gelu_t50", Workload("sh_dec", 55, 50, 1024, 1024, 6, 2, ACT_GELU, torch.bfloat16, True, 0.03,
                                 random_bias=True, n_shared=1, sel_s=0.4, zipf_s=0.4), None),
    ("few_router_n32", Workload("sh_few", 56, 40, 256, 128, 32, 8, ACT_SWIGLU, torch.bfloat16, False, 0.05,
                                zipf_s=0.4, n_shared=1, sel_s=0.9), None),
]


@pytest.mark.parametrize("name,wl,_", SHARED_CASES, ids=[c[0] for c in SHARED_CASES])
def test_shared_expert_and_selection_bias(name, wl, _):
    """DeepSeek-V3's shared expert and selection-only bias: the kept set follows the device's
    logits plus the bias (in fp32), the gate weights and statistics the raw scores, and the
    shared FFN is added after the routed sum; every router and GEMM family."""
    inp = make_inputs(wl, "cuda")
    layer, y, ws, aux, V, ref, errs = run_full(wl, inp)
    check_aux(aux, V, wl.N, wl.K)
    if wl.dtype == torch.bfloat16:
        y16, _, _ = layer.forward(y_dtype=torch.bfloat16, with_aux=False)
        assert torch.equal(y16, y.to(torch.bfloat16))


def test_selection_bias_balances_a_skewed_router():
    """With the selection bias equal and opposite to the Zipf router bias, the choice of experts
    is as balanced as without either bias, while the weights keep the skew."""
    base = Workload("bal", 57, 4000, 256, 128, 16, 2, ACT_SWIGLU, torch.bfloat16, False, 0.05)
    counts = {}
    for tag, wl in (("plain", base), ("skewed", base.with_(zipf_s=1.0)), ("balanced", base.with_(zipf_s=1.0,
                                                                                                  sel_s=1.0))):
        inp = make_inputs(wl, "cuda")
        layer = Layer(wl, inp)
        y, ws, aux = layer.forward()
        counts[tag] = aux["counts"].cpu().numpy()
    cv = {k: v.std() / v.mean() for k, v in counts.items()}
    assert cv["skewed"] > 3 * cv["plain"]
    assert cv["balanced"] < 1.5 * cv["plain"]


# ----------------------------------------------------------------------------- capacity (drop)
CAPACITY_CASES = [
    ("fp32_small_router", Workload("cap_f32", 60, 300, 64, 256, 8, 2, ACT_GELU, torch.float32, True, 0.05,
                                   zipf_s=1.0, random_bias=True, capacity_factor=1.0)),
    ("fp32_chunked_router", Workload("cap_f32c", 61, 2300, 64, 128, 16, 3, ACT_GELU, torch.float32, False, 0.05,
                                     zipf_s=0.8, capacity_factor=1.25)),
    ("bf16_simt_router_fused_k2", Workload("cap_k2", 62, 1500, 256, 512, 6, 2, ACT_GELU, torch.bfloat16, True, 0.04,
                                           zipf_s=1.0, random_bias=True, capacity_factor=1.0)),
    ("bf16_tc_router_k4", Workload("cap_tc", 63, 1200, 256, 256, 64, 4, ACT_SWIGLU, torch.bfloat16, False, 0.05,
                                   zipf_s=1.0, capacity_factor=0.75)),
    ("bf16_pairs_shared", Workload("cap_sh", 64, 1500, 512, 1024, 8, 2, ACT_SWIGLU, torch.bfloat16, False, 0.04,
                                   zipf_s=0.9, n_shared=1, capacity_factor=1.0)),
    ("decode8", WORKLOADS["decode8"].with_(zipf_s=2.0, capacity_factor=1.0)),
    ("decode64_bias", WORKLOADS["decode64"].with_(zipf_s=1.0, sel_s=0.5, capacity_factor=0.5)),
    ("huge_capacity", Workload("cap_big", 65, 700, 256, 256, 8, 2, ACT_SWIGLU, torch.bfloat16, False, 0.05,
                               zipf_s=0.5, capacity_factor=8.0)),
]


@pytest.mark.parametrize("name,wl", CAPACITY_CASES, ids=[c[0] for c in CAPACITY_CASES])
def test_capacity_drop(name, wl):
    """Per-expert capacity with drop: each expert's segment holds its first C assignments in token
    order (bit-exact against the oracle's decision on the device's routing), the dropped slots add
    nothing, and the statistics still describe the router's own choice."""
    inp = make_inputs(wl, "cuda")
    layer, y, ws, aux, V, ref, errs = run_full(wl, inp)
    check_aux(aux, V, wl.N, wl.K)
    C = ref["capacity"]
    assert C == int(np.ceil(ph.capacity_factor(wl) * wl.T * wl.K / wl.N))
    dropped = int((ref["keep"] == 0).sum())
    if name == "huge_capacity":
        assert dropped == 0
    else:
        assert dropped > 0, "the case should overflow some expert"


REROUTE_CASES = [
    ("fp32_small_router", Workload("rr_f32", 66, 300, 64, 256, 8, 2, ACT_GELU, torch.float32, True, 0.05,
                                   zipf_s=1.2, random_bias=True, capacity_factor=1.0, overflow=1)),
    ("fp32_chunked_router_k3", Workload("rr_f32c", 67, 2300, 64, 128, 16, 3, ACT_GELU, torch.float32, False, 0.05,
                                        zipf_s=1.0, capacity_factor=0.9, overflow=1)),
    ("bf16_simt_router_k2", Workload("rr_k2", 68, 1500, 256, 512, 6, 2, ACT_GELU, torch.bfloat16, True, 0.04,
                                     zipf_s=1.0, random_bias=True, capacity_factor=1.0, overflow=1)),
    ("bf16_tc_router_k8_bias", Workload("rr_tc", 69, 1200, 256, 256, 64, 8, ACT_SWIGLU, torch.bfloat16, False, 0.05,
                                        zipf_s=1.2, sel_s=0.3, capacity_factor=0.6, overflow=1)),
    ("bf16_shared", Workload("rr_sh", 70, 1500, 512, 1024, 8, 2, ACT_SWIGLU, torch.bfloat16, False, 0.04,
                             zipf_s=0.9, n_shared=1, capacity_factor=0.8, overflow=1)),
    ("decode8", WORKLOADS["decode8"].with_(zipf_s=2.0, capacity_factor=1.0, overflow=1)),
    ("decode64_bias", WORKLOADS["decode64"].with_(zipf_s=1.0, sel_s=0.5, capacity_factor=0.5, overflow=1)),
    ("huge_capacity", Workload("rr_big", 71, 700, 256, 256, 8, 2, ACT_SWIGLU, torch.bfloat16, False, 0.05,
                               zipf_s=0.5, capacity_factor=8.0, overflow=1)),
]


@pytest.mark.parametrize("name,wl", REROUTE_CASES, ids=[c[0] for c in REROUTE_CASES])
def test_capacity_reroute(name, wl):
    """Per-expert capacity with the next-candidate reroute: the expert serving every slot is the
    oracle's reroute decision on the device's selection values (bit-exact), each expert's segment
    holds its slots in token order, dropped slots add nothing, y matches the oracle, and the
    statistics still describe the router's own choice."""
    inp = make_inputs(wl, "cuda")
    layer = Layer(wl, inp)
    T, N, K = wl.T, wl.N, wl.K
    y, ws, aux = layer.forward()
    V = layer.views(ws, T)
    ref = ph.oracle_full_layer(inp, wl, K, gpu_logits=V["logits"])
    C = ref["capacity"]
    assert C == int(np.ceil(ph.capacity_factor(wl) * T * K / N))
    ph.assert_logits_close(V["logits"], ref["scores"])
    sel = oracle.select_topk(ph.selection_scores(V["logits"], inp).astype(np.float64), K)
    assign = oracle.capacity_reroute(ph.selection_scores(V["logits"], inp).astype(np.float64), sel, C)
    np.testing.assert_array_equal(assign, ref["assign"])
    # idx holds the serving expert; a dropped slot keeps its (full) selected expert
    np.testing.assert_array_equal(V["idx"], np.where(assign >= 0, assign, sel))
    ph.assert_weights_close(V["w"], ref["w"], ref["scores"])
    kept = assign.ravel() >= 0
    flat = assign.ravel()
    counts = np.bincount(flat[kept], minlength=N)
    assert (counts <= C).all()
    np.testing.assert_array_equal(V["counts"], counts)
    ro = V["row_offsets"]
    for e in range(N):
        seg = V["perm_slot"][ro[e]:ro[e] + counts[e]]
        np.testing.assert_array_equal(seg, np.nonzero(flat == e)[0])
    assert np.all(V["slot_row"][~kept] == -1)
    ph.assert_y_close(y.float().cpu().numpy(), ref["y"], wl.dtype)
    # statistics of the router's choice, before the capacity
    st = oracle.aux_stats(V["logits"].astype(np.float64), sel, V["w"].astype(np.float64), N)
    np.testing.assert_array_equal(aux["counts"].cpu().numpy(), st["counts"].astype(np.int32))
    rerouted = int(((assign != sel) & (assign >= 0)).sum())
    if name == "huge_capacity":
        assert rerouted == 0 and kept.all()
    else:
        assert rerouted > 0, "the case should reroute some slot"


# ----------------------------------------------------------------------------- expert parallelism
EP_CASES = [
    ("gelu_bias_2_ranks", Workload("ep_a", 80, 700, 256, 512, 8, 2, ACT_GELU, torch.bfloat16, True, 0.04,
                                   zipf_s=0.5, random_bias=True), 2),
    ("swiglu_64_experts_4_ranks", Workload("ep_b", 81, 600, 256, 256, 64, 4, ACT_SWIGLU, torch.bfloat16, False, 0.05,
                                           zipf_s=0.5, sel_s=0.3), 4),
    ("few_tokens_4_ranks", Workload("ep_c", 82, 24, 512, 512, 16, 4, ACT_SWIGLU, torch.bfloat16, False, 0.04,
                                    zipf_s=0.6), 4),
    ("fp32_2_ranks", Workload("ep_d", 83, 300, 64, 256, 8, 2, ACT_GELU, torch.float32, True, 0.05,
                              random_bias=True), 2),
    ("one_rank", Workload("ep_e", 84, 500, 256, 256, 8, 2, ACT_SWIGLU, torch.bfloat16, False, 0.05), 1),
]


@pytest.mark.parametrize("name,wl,R", EP_CASES, ids=[c[0] for c in EP_CASES])
def test_expert_parallel_virtual_ranks(name, wl, R):
    """Expert parallelism emulated on one GPU: R virtual ranks each route and pack their own
    tokens (moe_ep_dispatch), the all-to-alls are buffer copies, each rank's N/R experts run on
    the rows it received (moe_ep_experts), the outputs go back and each rank combines
    (moe_ep_combine).  Every rank's routing is bit-exact and its y equals the oracle's whole
    layer on its tokens with all N experts."""
    T, N, K, D = wl.T, wl.N, wl.K, wl.D
    epr = N // R
    big = make_inputs(wl, "cuda", T=T * R)
    cfg = moe.make_config(wl.D, wl.H, N, K, wl.act, moe.dtype_code(wl.dtype), wl.has_bias)
    w_router = moe.make_weights(big["W_g"], big["W1"], big["W2"], big["b_g"], big["b1"], big["b2"], big.get("b_sel"))
    L = moe.moe_get_workspace_layout(cfg, T)
    sent = []
    for r in range(R):
        x_r = big["x"][r * T:(r + 1) * T].contiguous()
        ws = torch.empty(moe.moe_ep_workspace_size(cfg, R, T), dtype=torch.uint8, device="cuda")
        send_x = torch.empty(T * K, D, dtype=wl.dtype, device="cuda")
        send_e = torch.full((T * K,), -1, dtype=torch.int32, device="cuda")
        send_w = torch.empty(T * K, device="cuda")
        cnt = torch.empty(R, dtype=torch.int32, device="cuda")
        pos = torch.empty(T * K, dtype=torch.int32, device="cuda")
        moe.check(moe.moe_ep_dispatch(cfg, R, x_r, T, w_router, send_x, send_e, send_w, cnt, pos, None, ws,
                                      ws.numel()), "dispatch")
        torch.cuda.synchronize()
        assert moe.moe_get_device_status() == 0
        lg = _ws_view(ws, L.logits, T * N, torch.float32).view(T, N).cpu().numpy()
        idx = _ws_view(ws, L.topk_idx, T * K, torch.int32).view(T, K).cpu().numpy()
        sent.append(dict(x=x_r, send_x=send_x, send_e=send_e, send_w=send_w, cnt=cnt.cpu().tolist(), pos=pos,
                         logits=lg, idx=idx))
        # the packing: rank-major, (token, slot) order inside a rank, nothing lost
        flat = idx.ravel()
        dest = flat // epr
        order = np.lexsort((np.arange(T * K), dest))
        np.testing.assert_array_equal(pos.cpu().numpy()[order], np.arange(T * K))
        np.testing.assert_array_equal(send_e.cpu().numpy()[pos.cpu().numpy()], flat - dest * epr)
        np.testing.assert_array_equal(np.bincount(dest, minlength=R), sent[-1]["cnt"])
    # the all-to-all, emulated: rank q receives every rank's block for q, source rank after source rank
    offs = [np.concatenate([[0], np.cumsum(s_["cnt"])]) for s_ in sent]
    z_parts = [[None] * R for _ in range(R)]
    for q in range(R):
        rx = torch.cat([s_["send_x"][offs[r][q]:offs[r][q + 1]] for r, s_ in enumerate(sent)])
        re = torch.cat([s_["send_e"][offs[r][q]:offs[r][q + 1]] for r, s_ in enumerate(sent)])
        rw = torch.cat([s_["send_w"][offs[r][q]:offs[r][q + 1]] for r, s_ in enumerate(sent)])
        M = rx.shape[0]
        cfg_l = moe.make_config(wl.D, wl.H, epr, 1, wl.act, moe.dtype_code(wl.dtype), wl.has_bias)
        sl = slice(q * epr, (q + 1) * epr)
        w_l = moe.make_weights(None, big["W1"][sl], big["W2"][sl], None,
                               None if big["b1"] is None else big["b1"][sl],
                               None if big["b2"] is None else big["b2"][sl])
        z = torch.full((max(M, 1), D), float("nan"), device="cuda")
        wsl = torch.empty(max(moe.moe_ep_experts_workspace_size(cfg_l, M), 1), dtype=torch.uint8, device="cuda")
        moe.check(moe.moe_ep_experts(cfg_l, rx, M, re, rw, w_l, z, wsl, wsl.numel()), "experts")
        torch.cuda.synchronize()
        assert moe.moe_get_device_status() == 0
        rstart = np.concatenate([[0], np.cumsum([s_["cnt"][q] for s_ in sent])])
        for r in range(R):
            z_parts[r][q] = z[rstart[r]:rstart[r + 1]]
    for r, s_ in enumerate(sent):
        z_back = torch.cat(z_parts[r]).contiguous()
        y = torch.full((T, D), float("nan"), device="cuda")
        moe.check(moe.moe_ep_combine(cfg, z_back, T, s_["pos"], y, moe.MOE_F32), "combine")
        torch.cuda.synchronize()
        inp_r = dict(big, x=s_["x"])
        ref = ph.oracle_full_layer(inp_r, wl, K, gpu_logits=s_["logits"])
        ph.assert_logits_close(s_["logits"], ref["scores"])
        np.testing.assert_array_equal(s_["idx"], ref["sel"])
        ph.assert_y_close(y.cpu().numpy(), ref["y"], wl.dtype)


# ----------------------------------------------------------------------------- backward
BACKWARD_CASES = [
    ("fp32_gelu_bias", Workload("bw_a", 90, 200, 64, 128, 8, 2, ACT_GELU, torch.float32, True, 0.05,
                                zipf_s=0.5, random_bias=True)),
    ("bf16_gelu_bias_simt_router", Workload("bw_b", 91, 300, 128, 256, 6, 2, ACT_GELU, torch.bfloat16, True, 0.05,
                                            zipf_s=0.5, random_bias=True)),
    ("bf16_swiglu_tc_router_bias", Workload("bw_c", 92, 260, 128, 192, 40, 4, ACT_SWIGLU, torch.bfloat16, False,
                                            0.05, zipf_s=0.4, sel_s=0.3)),
    ("bf16_swiglu_few_tokens", Workload("bw_d", 93, 20, 256, 128, 16, 3, ACT_SWIGLU, torch.bfloat16, False, 0.05,
                                        zipf_s=0.4)),
]


def _rel_l2(a, b):
    return float(np.linalg.norm(a.astype(np.float64) - b) / max(np.linalg.norm(b), 1e-300))


@pytest.mark.parametrize("name,wl", BACKWARD_CASES, ids=[c[0] for c in BACKWARD_CASES])
def test_backward_matches_oracle(name, wl):
    """The layer's backward (dx and every parameter's gradient, through the experts, the softmax
    over the kept scores and both trainable auxiliary losses) against the oracle's fp64 chain
    rule on the same routing.  The device computes in fp32 from the exact inputs, so every
    gradient is within relative L2 1e-4 and max-abs 1e-4 of its largest entry."""
    inp = make_inputs(wl, "cuda")
    T, D, H, N, K = wl.T, wl.D, wl.H, wl.N, wl.K
    layer = Layer(wl, inp)
    y, ws_f, _ = layer.forward(with_aux=False)
    V = layer.views(ws_f, T)
    g = torch.Generator(device="cuda").manual_seed(7)
    dy = torch.randn(T, D, generator=g, device="cuda")
    rows1 = 2 * H if wl.act == ACT_SWIGLU else H
    gr = dict(dx=torch.full((T, D), float("nan"), device="cuda"), dW_g=torch.full((D, N), float("nan"), device="cuda"),
              db_g=torch.full((N,), float("nan"), device="cuda"),
              dW1=torch.full((N, rows1, D), float("nan"), device="cuda"),
              dW2=torch.full((N, D, H), float("nan"), device="cuda"))
    if wl.has_bias:
        gr["db1"] = torch.full((N, H), float("nan"), device="cuda")
        gr["db2"] = torch.full((N, D), float("nan"), device="cuda")
    ws = torch.empty(moe.moe_backward_workspace_size(layer.cfg, T), dtype=torch.uint8, device="cuda")
    a_s, a_i = 0.6, 1.7
    moe.check(moe.moe_backward(layer.cfg, inp["x"], T, layer.w, dy, a_s, a_i, moe.make_grads(**gr), ws, ws.numel()),
              "backward")
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == 0
    ref = oracle.moe_layer_backward(ph.host(inp["x"]), ph.host(inp["W_g"]), ph.host(inp["W1"]), ph.host(inp["W2"]),
                                    dy.cpu().numpy().astype(np.float64), K=K, act=wl.act, dtype_tag=ph.tag(wl.dtype),
                                    bg=ph.host(inp["b_g"]), b1=ph.host(inp["b1"]), b2=ph.host(inp["b2"]),
                                    bsel=ph.host(inp.get("b_sel")),
                                    sel_scores=ph.selection_scores(V["logits"], inp), alpha_switch=a_s,
                                    alpha_importance=a_i)
    pairs = [("dx", "dx"), ("dW_g", "dWg"), ("db_g", "dbg"), ("dW1", "dW1"), ("dW2", "dW2")]
    if wl.has_bias:
        pairs += [("db1", "db1"), ("db2", "db2")]
    for mine, theirs in pairs:
        a = gr[mine].cpu().numpy()
        b = ref[theirs]
        assert np.all(np.isfinite(a)), mine
        assert _rel_l2(a, b) <= 1e-4, (mine, _rel_l2(a, b))
        assert np.abs(a - b).max() <= 1e-4 * max(np.abs(b).max(), 1e-30), mine
    # the same gradients twice, bit for bit
    gr2 = {k: torch.empty_like(v) for k, v in gr.items()}
    moe.check(moe.moe_backward(layer.cfg, inp["x"], T, layer.w, dy, a_s, a_i, moe.make_grads(**gr2), ws, ws.numel()))
    torch.cuda.synchronize()
    for k in gr:
        assert torch.equal(gr[k], gr2[k]), k


# ----------------------------------------------------------------------------- data parallelism
def _ws_view(ws, off, n, dt):
    return ws[off:off + n * torch.tensor([], dtype=dt).element_size()].view(dt)


@pytest.mark.parametrize("name,T0,T1", [("gpt2", 700, 333), ("tiny", 200, 77), ("many", 300, 129)])
def test_data_parallel_statistics_from_two_shards(name, T0, T1):
    """Token-sharded data parallelism emulated on one GPU: each shard's layer call leaves its
    routing in its workspace, moe_aux_partials exports exact integer sums, their sum is
    finalised, and the statistics equal the oracle's over the union batch.  The fixed-point
    sums equal their definition exactly, and the device and host finalisations give the
    same bits."""
    if name == "many":
        wl = Workload("many_dp", 40, T0 + T1, 256, 128, 64, 4, ACT_SWIGLU, torch.bfloat16, False, 0.05,
                      zipf_s=0.5)
    else:
        wl = WORKLOADS[name]
    inp = make_inputs(wl, "cuda", T=T0 + T1)
    layer = Layer(wl, inp)
    N, K = wl.N, wl.K
    parts, routed = [], []
    for a, b in ((0, T0), (T0, T0 + T1)):
        T = b - a
        x = inp["x"][a:b].contiguous()
        y, ws, _ = layer.forward(x=x, with_aux=False)
        L = moe.moe_get_workspace_layout(layer.cfg, T)
        lg = _ws_view(ws, L.logits, T * N, torch.float32)
        idx = _ws_view(ws, L.topk_idx, T * K, torch.int32)
        w = _ws_view(ws, L.topk_w, T * K, torch.float32)
        part = torch.full((moe.aux_partials_len(N),), -7, dtype=torch.int64, device="cuda")
        moe.check(moe.moe_aux_partials(layer.cfg, T, lg, idx, w, part), "partials")
        torch.cuda.synchronize()
        assert moe.moe_get_device_status() == 0
        parts.append(part)
        routed.append((lg.view(T, N).cpu().numpy(), idx.view(T, K).cpu().numpy(), w.view(T, K).cpu().numpy()))
    lg = np.concatenate([r[0] for r in routed])
    sel = np.concatenate([r[1] for r in routed])
    w = np.concatenate([r[2] for r in routed])
    total = parts[0] + parts[1]          # the all-reduce of two ranks
    p = total.cpu().numpy()
    fixed = np.rint(w.astype(np.float64) * 4294967296.0).astype(np.int64)
    np.testing.assert_array_equal(p[:N], np.bincount(sel.ravel(), minlength=N))
    np.testing.assert_array_equal(p[N:2 * N], np.array([fixed[sel == e].sum() for e in range(N)]))
    assert p[3 * N] == T0 + T1
    out = dict(counts=torch.full((N,), -1, dtype=torch.int32, device="cuda"),
               importance=torch.full((N,), -1.0, device="cuda"), p_mean=torch.full((N,), -1.0, device="cuda"),
               scalars=torch.full((4,), -1.0, device="cuda"))
    moe.check(moe.moe_aux_finalize(layer.cfg, total, moe.make_aux(**out)), "finalize")
    torch.cuda.synchronize()
    host = dict(counts=torch.empty(N, dtype=torch.int32), importance=torch.empty(N), p_mean=torch.empty(N),
                scalars=torch.empty(4))
    moe.check(moe.moe_aux_finalize_host(layer.cfg, total.cpu(), **host), "finalize host")
    for k in out:
        assert torch.equal(out[k].cpu(), host[k]), k
    st = oracle.aux_stats(lg.astype(np.float64), sel, w.astype(np.float64), N)
    np.testing.assert_array_equal(out["counts"].cpu().numpy(), st["counts"].astype(np.int32))
    np.testing.assert_allclose(out["importance"].cpu().numpy(), st["importance"], rtol=1e-6, atol=1e-6)
    np.testing.assert_allclose(out["p_mean"].cpu().numpy(), st["p_mean"], rtol=1e-5, atol=1e-7)
    np.testing.assert_allclose(out["scalars"].cpu().numpy(),
                               [st["switch"], st["simple"], st["cv2_importance"], st["cv2_load"]], rtol=1e-4, atol=1e-6)


# ----------------------------------------------------------------------------- entry points, determinism
def test_route_entry_point_matches_forward():
    wl = WORKLOADS["gpt2"]
    inp = make_inputs(wl, "cuda", T=500)
    layer = Layer(wl, inp)
    y, ws, aux = layer.forward()
    V = layer.views(ws, 500)
    logits = torch.empty(500, wl.N, device="cuda")
    idx = torch.empty(500, wl.K, dtype=torch.int32, device="cuda")
    w = torch.empty(500, wl.K, device="cuda")
    cnt = torch.empty(wl.N, dtype=torch.int32, device="cuda")
    ws2 = moe.alloc_workspace(layer.cfg, 500)
    moe.check(moe.moe_route(layer.cfg, inp["x"], 500, layer.w, logits, idx, w, cnt, ws2, ws2.numel()))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(logits.cpu().numpy(), V["logits"])
    np.testing.assert_array_equal(idx.cpu().numpy(), V["idx"])
    np.testing.assert_array_equal(w.cpu().numpy(), V["w"])
    np.testing.assert_array_equal(cnt.cpu().numpy(), V["counts"])
    out = dict(counts=torch.empty(wl.N, dtype=torch.int32, device="cuda"), importance=torch.empty(wl.N, device="cuda"),
               p_mean=torch.empty(wl.N, device="cuda"), scalars=torch.empty(4, device="cuda"))
    moe.check(moe.moe_aux_stats(layer.cfg, 500, logits, idx, w, moe.make_aux(**out), ws2, ws2.numel()))
    torch.cuda.synchronize()
    # the layer computes its statistics inside the router kernel, moe_aux_stats in its own kernels:
    # counts are equal, the float sums agree to rounding (different fixed summation orders)
    assert torch.equal(out["counts"], aux["counts"])
    for k in ("importance", "p_mean", "scalars"):
        torch.testing.assert_close(out[k], aux[k], rtol=1e-5, atol=1e-6)


def test_bitwise_deterministic_runs():
    for name, T in [("gpt2", 2000), ("mixtral", 300), ("decode1", 1), ("decode8", 8)]:
        wl = WORKLOADS[name]
        inp = make_inputs(wl, "cuda", T=T)
        layer = Layer(wl, inp)
        y1, ws1, a1 = layer.forward()
        y2, ws2, a2 = layer.forward()
        assert torch.equal(y1, y2)
        for k in a1:
            assert torch.equal(a1[k], a2[k])
        del inp, layer
        torch.cuda.empty_cache()


CANARY_CASES = [("tiny", 300), ("gpt2", 2000), ("mixtral", 300), ("decode1", 1), ("decode8", 8),
                ("deepseek_zipf", 1024)]


@pytest.mark.parametrize("name,T", CANARY_CASES, ids=[f"{c[0]}_T{c[1]}" for c in CANARY_CASES])
def test_workspace_and_output_canaries(name, T):
    """Nothing is written outside the buffers a call is given: the workspace is embedded in a larger
    buffer whose guard bytes (a byte pattern before and after it) must survive the layer call, and so
    must the guard rows around y."""
    wl = WORKLOADS[name]
    if name.startswith("deepseek"):
        wl = wl.with_(N=32)   # the DeepSeek-shaped layer with 32 experts (2.8 GB of weights)
    inp = make_inputs(wl, "cuda", T=T)
    layer = Layer(wl, inp)
    n = moe.moe_workspace_size(layer.cfg, T)
    guard = 1 << 16
    big = torch.full((n + 2 * guard,), 0xA5, dtype=torch.uint8, device="cuda")
    ws = big[guard:guard + n]
    assert ws.data_ptr() % 256 == 0
    yb = torch.full((T + 2, wl.D), 7.25, device="cuda")
    y = yb[1:T + 1]
    aux = dict(counts=torch.empty(wl.N, dtype=torch.int32, device="cuda"), importance=torch.empty(wl.N, device="cuda"),
               p_mean=torch.empty(wl.N, device="cuda"), scalars=torch.empty(4, device="cuda"))
    moe.check(moe.moe_forward(layer.cfg, inp["x"], T, layer.w, y, moe.MOE_F32, moe.make_aux(**aux), ws, n))
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == 0
    assert bool((big[:guard] == 0xA5).all()) and bool((big[guard + n:] == 0xA5).all())
    assert bool((yb[0] == 7.25).all()) and bool((yb[T + 1] == 7.25).all())
    assert torch.isfinite(y).all()
    del inp, layer, big
    torch.cuda.empty_cache()


def test_nan_scores_rank_last_and_flag_status():
    wl = WORKLOADS["tiny"]
    inp = make_inputs(wl, "cuda", T=64)
    inp["x"][7, 3] = float("nan")
    layer = Layer(wl, inp)
    ws = moe.alloc_workspace(layer.cfg, 64)
    y = torch.empty(64, wl.D, device="cuda")
    moe.check(moe.moe_forward(layer.cfg, inp["x"], 64, layer.w, y, moe.MOE_F32, None, ws, ws.numel()))
    st = moe.moe_get_device_status()
    assert st & moe.MOE_STATUS_NAN_LOGIT
    V = layer.views(ws, 64)
    assert V["idx"][7].tolist() == [0, 1]  # every score NaN -> all rank as -inf -> lowest indices
    ok = np.ones(64, bool)
    ok[7] = False
    ref = ph.oracle_full_layer(inp | {"x": inp["x"][torch.from_numpy(ok).cuda()]}, wl, wl.K,
                               gpu_logits=V["logits"][ok])
    ph.assert_y_close(y[torch.from_numpy(ok).cuda()].cpu().numpy(), ref["y"], wl.dtype)
    assert moe.moe_get_device_status() == 0


def test_bounded_wait_expires_and_context_survives():
    moe.check(moe.moe_selftest_wait_timeout(20_000_000))
    st = moe.moe_get_device_status()
    assert st & moe.MOE_STATUS_TIMEOUT
    assert moe.moe_get_device_status() == 0
    wl = WORKLOADS["tiny"]
    run_full(wl, make_inputs(wl, "cuda", T=64))
