"""GPU parity: the CUDA path, called through the C ABI, against the CPU oracle.

Bit-exact: Eq. (6) codes and scales, activation codes and scales, routing
(outside the 1e-5 router-margin band), counts, offsets, the permutation and
every INT32 group partial.  Within tolerance: gates (relative error at most
twice the largest logit difference plus 1e-6), SwiGLU
codes (equal or one apart near a rounding boundary) and y
(max|dy| <= 2e-3 max|y_ref|)."""
import numpy as np
import pytest
import torch

import oracle
from moe_ffn_layer_fp32_b200 import _lib, synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

_CACHE = {}


def workload(name):
    if name not in _CACHE:
        w = synth.WORKLOADS[name]
        q = oracle.quantize_layer(synth.workload_layer(w))
        _CACHE[name] = (w, q)
    return _CACHE[name]


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    gu.ensure_built()


# ---------------------------------------------------------------------------
def test_quantizer_matches_oracle_bit_exact():
    from moe_ffn_layer_fp32_b200.layer import quantize_int4
    rng = np.random.default_rng(0)
    W = (rng.standard_normal((513, 512)) * 0.02).astype(np.float32)
    W[7] = 0.0
    W[8, :32] = np.float32(7.5) * np.float32(2.0 ** -6)
    W[9, 5] = 1e-30
    W[10] = rng.standard_normal(512).astype(np.float32) * 1e4
    for name in ("eq6_int4_cases.txt",):
        from tests.conftest import read_cases
        for i, c in enumerate(read_cases(name)):
            W[20 + i, :32] = c["w"].astype(np.float32)
    p_gpu, s_gpu = quantize_int4(torch.from_numpy(W).cuda())
    p_ref, s_ref = oracle.quantize_int4(W)
    assert np.array_equal(p_gpu.cpu().numpy(), p_ref)
    assert np.array_equal(s_gpu.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


def _full_check(q, x, deterministic=False, partial_rows=None, max_tokens=None, cuda_cores=False, decode=True,
                atomic_combine=False, tc_int8=False, fused_decode=True, fused_requant=False):
    T = x.shape[0]
    L = gu.make_gpu_layer(q, max_tokens or max(T, 1), deterministic=deterministic, cuda_cores=cuda_cores,
                          decode=decode, atomic_combine=atomic_combine, tc_int8=tc_int8, fused_decode=fused_decode,
                          fused_requant=fused_requant)
    out = gu.run_gpu(L, q, x)
    y, D = oracle.moe_layer(q, x, dumps=True)
    rep = {}
    assert np.array_equal(out["xq"], D["xq"]) and np.array_equal(out["sx"].view(np.uint32), D["sx"].view(np.uint32))
    assert np.max(np.abs(out["logits"] - D["logits"])) <= gu.LOGIT_TOL * max(1.0, np.abs(D["logits"]).max())
    gu.check_routing_and_permutation(q, out, D["idx"], D["gate"], D["probs"], rep, D["logits"])
    gu.check_hq(q, out, D, rep)
    gu.check_y(out["y"], y, rep)
    if partial_rows is not None:
        gu.check_partials(L, q, out, partial_rows)
    L.close()
    return rep, out


@pytest.mark.parametrize("path", ["decode", "tensor_cores", "tensor_cores_i8", "cuda_cores"])
@pytest.mark.parametrize("combine", ["atomic", "fixed_order"])
def test_c0_all_stages(combine, path):
    # T = 64 takes the decode kernels by default; the others force the prefill kernels: the
    # kind::f16 tensor-core GEMMs (default), the kind::i8 ones, or the CUDA-core ones.
    # atomic: the decode path's default, forced on the prefill path; fixed_order: forced on the decode path
    w, q = workload("c0")
    x = synth.workload_x(w)
    R = w.T * (q.k + 1)
    rep, out = _full_check(q, x, combine == "fixed_order", partial_rows=range(0, R, 3),
                           cuda_cores=path == "cuda_cores", decode=path == "decode",
                           atomic_combine=combine == "atomic", tc_int8=path == "tensor_cores_i8")
    print("c0", path, rep)


def test_deterministic_mode_is_reproducible():
    w, q = workload("c0")
    x = synth.workload_x(w)
    L = gu.make_gpu_layer(q, w.T, deterministic=True)
    a = gu.run_gpu(L, q, x, stages=False)["y"]
    b = gu.run_gpu(L, q, x, stages=False)["y"]
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


@pytest.mark.parametrize("T,decode", [(T, True) for T in (1, 2, 7, 31, 33, 63, 64, 65, 127, 129, 300)]
                         + [(T, False) for T in (1, 7, 33, 64)])
def test_ragged_token_counts(T, decode):
    w, q = workload("c0")
    x = synth.draw_x(T, w.d, seed=100 + T)
    rep, out = _full_check(q, x, max_tokens=512, partial_rows=[0, T * q.k - 1, T * q.k, T * (q.k + 1) - 1],
                           decode=decode)
    assert out["counts"][q.E] == T


@pytest.mark.parametrize("T", [1, 2, 5, 8])
@pytest.mark.parametrize("fused", [True, False], ids=["one_launch", "four_launches"])
def test_small_decode_batches_both_kernel_sets(T, fused):
    # up to 8 tokens run as one launch of clusters by default; the four-launch kernels give the same
    # results
    w, q = workload("c0")
    x = synth.draw_x(T, w.d, seed=200 + T)
    R = T * (q.k + 1)
    rep, out = _full_check(q, x, max_tokens=64, partial_rows=range(R), fused_decode=fused)
    assert out["counts"][q.E] == T


@pytest.mark.parametrize("T", [1, 8])
def test_c1_decode_one_launch_matches_four_launches(T):
    # the decode workload's shapes (d_model 1024, hidden 512): both kernel sets against the oracle,
    # and against each other (the same expert outputs, added into y in a different order)
    w = synth.WORKLOADS["c1"]
    q = oracle.quantize_layer(synth.workload_layer(w, 5))
    x = synth.workload_x(w, step=5, T=T)
    _, a = _full_check(q, x, max_tokens=64, fused_decode=True)
    _, b = _full_check(q, x, max_tokens=64, fused_decode=False)
    assert np.array_equal(a["idx"], b["idx"]) and np.array_equal(a["hq"], b["hq"])
    assert np.max(np.abs(a["y"] - b["y"])) <= 1e-5 * np.abs(b["y"]).max()


@pytest.mark.parametrize("name,T", [("c0", 1), ("c0", 3), ("c0", 8), ("s2048", 1), ("s2048", 8), ("c4dec", 1),
                                    ("c4dec", 2), ("c4dec", 8)])
def test_one_launch_decode_against_four_launches(name, T):
    # The one-launch decode (clusters of 8 CTAs; of 16 for one or two tokens on the d_model 2048 /
    # hidden 1024 shape) against the oracle, and against the four-launch path with its fixed-order
    # combine: the same routing, the same SwiGLU codes and scales bit for bit; y within 1e-5 of it
    # (the two routers add the FP32 products in different orders, so gates may differ in the last bits).
    w, q = workload(name)
    x = synth.draw_x(T, w.d, seed=300 + T)
    _, a = _full_check(q, x, max_tokens=64, fused_decode=True, partial_rows=[0, T * q.k - 1, T * q.k])
    _, b = _full_check(q, x, max_tokens=64, fused_decode=False, deterministic=True)
    assert np.array_equal(a["idx"], b["idx"]) and np.array_equal(a["slot_row"], b["slot_row"])
    assert np.max(np.abs(a["gate"] - b["gate"]) / np.abs(b["gate"])) <= 1e-5
    assert np.array_equal(a["hq"], b["hq"]) and np.array_equal(a["sh"].view(np.uint32), b["sh"].view(np.uint32))
    assert np.max(np.abs(a["y"] - b["y"])) <= 1e-5 * np.abs(b["y"]).max()


@pytest.mark.parametrize("name", ["c0", "c1", "s2048", "c4dec"])
def test_one_launch_decode_taken(name):
    # a forward of up to 8 tokens is one launch of the one-launch decode on every workload shape
    w = synth.WORKLOADS[name]
    from moe_ffn_layer_fp32_b200.layer import MoELayer
    L = MoELayer(w.d, w.h, shared_hidden=w.hs, n_experts=w.E, top_k=w.k, max_tokens=64)
    q = oracle.quantize_layer(synth.workload_layer(w))
    L.load(q.w_router, q.router_bias, q.w_gate_up, q.s_gate_up, q.w_down, q.s_down)
    x = gu.x_to_device(synth.draw_x(3, w.d, seed=7))
    L.profile(True)
    L.forward(x)
    torch.cuda.synchronize()
    launches = {k: v[0] for k, v in L.profile_read().items() if v[0]}
    L.close()
    assert launches == {"decode_fused": 1}, launches


def test_one_launch_decode_deterministic_and_repeatable():
    # in deterministic mode y of the one-launch decode is added in a fixed order: repeated calls agree
    # bit for bit, and the contribution counters left by each call let the next one (of another size)
    # combine correctly
    w, q = workload("c0")
    L = gu.make_gpu_layer(q, 64, deterministic=True)
    for T in (8, 1, 8, 5):
        x = synth.draw_x(T, w.d, seed=400 + T)
        y1 = gu.run_gpu(L, q, x, stages=False)["y"]
        y2 = gu.run_gpu(L, q, x, stages=False)["y"]
        assert np.array_equal(y1.view(np.uint32), y2.view(np.uint32))
        rep = {}
        gu.check_y(y1, oracle.moe_layer(q, x), rep)
    L.close()


def test_one_launch_decode_atomics_repeated_calls():
    # by default the one-launch decode clears y and adds the gate-weighted rows with atomics: calls of
    # changing size (each leaving its counters for the next) all match the oracle, and repeated calls
    # agree within FP32 rounding of the summation order
    w, q = workload("c0")
    L = gu.make_gpu_layer(q, 64)
    for T in (8, 1, 8, 5, 2):
        x = synth.draw_x(T, w.d, seed=410 + T)
        y1 = gu.run_gpu(L, q, x, stages=False)["y"]
        y2 = gu.run_gpu(L, q, x, stages=False)["y"]
        y_or = oracle.moe_layer(q, x)
        rep = {}
        gu.check_y(y1, y_or, rep)
        assert np.max(np.abs(y1 - y2)) <= 1e-5 * np.abs(y_or).max()
    L.close()


@pytest.mark.parametrize("T,decode,fused", [(3, True, True), (20, True, False), (200, False, False)],
                         ids=["one_launch", "four_launches", "prefill"])
def test_routing_ties_lowest_index_wins(T, decode, fused):
    # experts 3 and 35 get identical router columns (a tie across the two halves of a warp's lanes), as
    # do 40 and 50 (within one half), both columns scaled up so that the pairs lead the ranking: every
    # router adds a column's products the same way for both experts of a pair, so their keys are equal
    # and the lower index must come first, exactly as in the oracle
    w = synth.WORKLOADS["c0"]
    lw = synth.draw_layer(w.d, w.h, seed=91)
    col_a, col_b = lw.w_router[:, 3] * 8, lw.w_router[:, 40] * 6
    lw.w_router[:, 3], lw.w_router[:, 35] = col_a, col_a
    lw.w_router[:, 40], lw.w_router[:, 50] = col_b, col_b
    q = oracle.quantize_layer(lw)
    x = synth.draw_x(T, w.d, seed=92)
    L = gu.make_gpu_layer(q, T, decode=decode, fused_decode=fused)
    out = gu.run_gpu(L, q, x, stages=False)
    L.close()
    _, _, idx_or, gate_or = oracle.router(q, x)
    assert np.array_equal(out["idx"], idx_or)
    for lo, hi in ((3, 35), (40, 50)):
        both = [t for t in range(T) if lo in idx_or[t] and hi in idx_or[t]]
        assert len(both) >= max(1, T // 16), (lo, hi, len(both))
        for t in both:
            r = list(out["idx"][t])
            assert r.index(lo) + 1 == r.index(hi)
            assert out["gate"][t][r.index(lo)] == out["gate"][t][r.index(hi)]


def test_decode_hot_groups_of_64_rows():
    # every token to experts 5, 9, 33, 58: four routed groups of 64 rows each (8 token blocks of the decode GEMV)
    w = synth.WORKLOADS["c0"]
    lw = synth.draw_layer(w.d, w.h, seed=44, bias_coef=None)
    lw.router_bias = np.full(60, -30.0, np.float32)
    lw.router_bias[[5, 9, 33, 58]] = 0.0
    q = oracle.quantize_layer(lw)
    x = synth.draw_x(64, w.d, seed=45)
    rep, out = _full_check(q, x, partial_rows=[0, 63, 64, 255, 256, 319])
    assert out["counts"][[5, 9, 33, 58]].tolist() == [64] * 4


@pytest.mark.parametrize("decode", [True, False], ids=["decode", "prefill"])
def test_top8_of_16_experts_64_tokens(decode):
    # top-8: 512 routing slots at T = 64 (two scatter rounds in the decode router's permutation)
    lw = synth.draw_layer(256, 128, E=16, seed=48)
    q = oracle.quantize_layer(lw, k=8)
    x = synth.draw_x(64, 256, seed=49)
    rep, out = _full_check(q, x, partial_rows=[0, 100, 511, 512, 575], decode=decode)
    assert out["counts"][:16].sum() == 512


def test_decode_every_expert_selected():
    # k = E: every token runs every routed expert (the full mixture)
    lw = synth.draw_layer(256, 128, E=4, seed=50)
    q = oracle.quantize_layer(lw, k=4)
    x = synth.draw_x(33, 256, seed=51)
    rep, out = _full_check(q, x, partial_rows=[0, 131, 132, 164])
    assert out["counts"].tolist() == [33] * 5


def test_decode_shared_expert_wider_than_routed():
    lw = synth.draw_layer(256, 64, seed=46, shared_hidden=256)
    q = oracle.quantize_layer(lw)
    x = synth.draw_x(40, 256, seed=47)
    rep, out = _full_check(q, x, partial_rows=[0, 77, 159, 160, 199])


def test_c2_prefill_cuda_cores():
    w, q = workload("c2")
    x = synth.workload_x(w, T=512)
    rep, out = _full_check(q, x, cuda_cores=True, partial_rows=[0, 2047, 2048, 2559])


def test_c2_prefill_atomic_combine():
    w, q = workload("c2")
    x = synth.workload_x(w, T=1024)
    rep, out = _full_check(q, x, atomic_combine=True, partial_rows=[0, 4095, 4096, 5119])


def test_T0_is_a_noop():
    w, q = workload("c0")
    L = gu.make_gpu_layer(q, 8)
    y = torch.full((1, w.d), 7.0, device="cuda")
    L.forward(torch.zeros((0, w.d), dtype=torch.bfloat16, device="cuda"), y[:0])
    torch.cuda.synchronize()
    assert torch.all(y == 7.0)


def test_skewed_routing_empty_and_hot_experts():
    # a bias that sends every token to experts 5, 9, 33, 58: 56 experts get no rows
    w = synth.WORKLOADS["c0"]
    lw = synth.draw_layer(w.d, w.h, seed=40, bias_coef=None)
    lw.router_bias = np.full(60, -30.0, np.float32)
    lw.router_bias[[5, 9, 33, 58]] = 0.0
    q = oracle.quantize_layer(lw)
    x = synth.draw_x(200, w.d, seed=41)
    rep, out = _full_check(q, x, partial_rows=[0, 199, 200, 799, 800, 999])
    assert sorted(np.nonzero(out["counts"][:60])[0].tolist()) == [5, 9, 33, 58]


def test_sigmoid_topk_normalised_gating():
    w = synth.WORKLOADS["c0"]
    q = oracle.quantize_layer(synth.workload_layer(w), gating=1)
    x = synth.workload_x(w)
    rep, out = _full_check(q, x)
    assert np.allclose(out["gate"].sum(axis=1), 1.0, atol=1e-6)


@pytest.mark.parametrize("decode,T", [(True, 64), (False, 200)], ids=["decode", "prefill"])
def test_selection_only_bias_gating(decode, T):
    # gating 2: the router bias (auxiliary-loss-free balancing) moves the top-k of the sigmoid
    # scores and enters no gate; the gates of a token sum to one
    w = synth.WORKLOADS["c0"]
    lw = synth.draw_layer(w.d, w.h, seed=60, bias_coef=0.25)
    q = oracle.quantize_layer(lw, gating=2)
    x = synth.draw_x(T, w.d, seed=61)
    R = T * (q.k + 1)
    rep, out = _full_check(q, x, decode=decode, partial_rows=[0, T * q.k - 1, T * q.k, R - 1])
    assert np.allclose(out["gate"].sum(axis=1), 1.0, atol=1e-6)
    print("selection bias", "decode" if decode else "prefill", rep)


def _group_edge_rows(out, E):
    """First and last row of every group that has rows (the shared group included)."""
    off = out["offsets"]
    rows = []
    for g in range(E + 1):
        if off[g + 1] > off[g]:
            rows += [int(off[g]), int(off[g + 1]) - 1]
    return sorted(set(rows))


@pytest.mark.parametrize("decode,T", [(True, 1), (True, 8), (True, 64), (False, 300)],
                         ids=["decode1", "decode8", "decode64", "prefill300"])
def test_mobilemoe_s_shape(decode, T):
    # the MobileMoE-S layer: d_model 768, 60 experts of hidden 384, shared expert hidden 1536 (4x)
    w, q = workload("s2048")
    x = synth.workload_x(w, T=T)
    L = gu.make_gpu_layer(q, max(T, 1), decode=decode)
    out = gu.run_gpu(L, q, x)
    y, D = oracle.moe_layer(q, x, dumps=True)
    rep = {}
    assert np.array_equal(out["xq"], D["xq"])
    gu.check_routing_and_permutation(q, out, D["idx"], D["gate"], D["probs"], rep, D["logits"])
    gu.check_hq(q, out, D, rep)
    gu.check_y(out["y"], y, rep)
    gu.check_partials(L, q, out, _group_edge_rows(out, q.E))
    L.close()
    print("s shape", T, rep)


def test_mobilemoe_s_prefill_2048():
    w, q = workload("s2048")
    x = synth.workload_x(w)
    L = gu.make_gpu_layer(q, w.T)
    out = gu.run_gpu(L, q, x)
    y, D = oracle.moe_layer(q, x, dumps=True)
    rep = {}
    gu.check_routing_and_permutation(q, out, D["idx"], D["gate"], D["probs"], rep, D["logits"])
    gu.check_hq(q, out, D, rep)
    gu.check_y(out["y"], y, rep)
    gu.check_partials(L, q, out, _group_edge_rows(out, q.E))
    L.close()
    print("s2048", rep)


@pytest.mark.parametrize("name,T", [("c0", 200), ("c2", 1024), ("c3b", 600)])
def test_prefill_fused_requantisation(name, T):
    # MMOE_FLAG_FUSED_REQUANT: the gate/up GEMM's clusters (1, 4 and 6 CTAs here) exchange the
    # per-token maxima and write the SwiGLU codes themselves
    w, q = workload(name)
    x = synth.workload_x(w, T=T)
    R = T * (q.k + 1)
    rep, out = _full_check(q, x, fused_requant=True, partial_rows=[0, T * q.k - 1, T * q.k, R - 1])
    print("fused requant", name, rep)


def test_c2_prefill_int8_tensor_cores():
    # the kind::i8 GEMMs (MMOE_FLAG_TC_INT8) on the balanced prefill workload
    w, q = workload("c2")
    x = synth.workload_x(w, T=1024)
    rep, out = _full_check(q, x, tc_int8=True, partial_rows=[0, 4095, 4096, 5119])


def test_shared_expert_wider_than_routed():
    # MobileMoE's shared expert is 4x a routed expert (final-architecture paragraph)
    lw = synth.draw_layer(256, 64, seed=42, shared_hidden=256)
    q = oracle.quantize_layer(lw)
    x = synth.draw_x(70, 256, seed=43)
    rep, out = _full_check(q, x, partial_rows=[0, 100, 279, 280, 349])


def test_forward_host_matches_device():
    w, q = workload("c0")
    x = synth.workload_x(w)
    L = gu.make_gpu_layer(q, w.T, deterministic=True)
    a = gu.run_gpu(L, q, x, stages=False)["y"]
    b = L.forward_host(x)
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


@pytest.mark.parametrize("pinned", [True, False])
def test_forward_host_chunked_equals_one_forward(pinned):
    # 3 * 8192 + 77 tokens: the host entry point splits the batch into three
    # chunks whose copies overlap the layer; y must equal one unsplit forward.
    w, q = workload("c0")
    T = 3 * 8192 + 77
    x = synth.workload_x(w, T=T)
    L = gu.make_gpu_layer(q, T, deterministic=True)
    a = gu.run_gpu(L, q, x, stages=False)["y"]
    if pinned:
        hx = torch.empty((T, w.d), dtype=torch.int16, pin_memory=True)
        hx.numpy()[:] = x.view(np.int16)
        hy = torch.full((T, w.d), float("nan"), dtype=torch.float32, pin_memory=True)
        b = L.forward_host(hx.numpy().view(np.uint16), hy.numpy())
    else:
        b = L.forward_host(x)
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    # the stream passed in is ordered after the copies: a device forward right after sees its own x
    c = gu.run_gpu(L, q, x[:100], stages=False)["y"]
    assert np.array_equal(c.view(np.uint32), a[:100].view(np.uint32))


def test_errors_on_device():
    w, q = workload("c0")
    from moe_ffn_layer_fp32_b200.layer import MoELayer
    L = MoELayer(q.d, q.h, max_tokens=8)
    x = torch.zeros((4, w.d), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(_lib.MMoEError) as ei:
        L.forward(x)
    assert ei.value.status == 2  # NOT_LOADED
    L.load(q.w_router, q.router_bias, q.w_gate_up, q.s_gate_up, q.w_down, q.s_down)
    with pytest.raises(_lib.MMoEError) as ei:
        L.forward(torch.zeros((9, w.d), dtype=torch.bfloat16, device="cuda"))
    assert ei.value.status == 1
    L.forward(x)
    with pytest.raises(_lib.MMoEError):
        L.stage(_lib.STAGE_SX, (9,), torch.float32)
    with pytest.raises(_lib.MMoEError):
        L.partials(0, 0, 100)


# --- the benchmark workloads ------------------------------------------------
def test_c1_decode_layers():
    w = synth.WORKLOADS["c1"]
    for layer in (0, 23):
        q = oracle.quantize_layer(synth.workload_layer(w, layer))
        for T in (1, 8):
            x = synth.workload_x(w, step=layer, T=T)
            rep, _ = _full_check(q, x, max_tokens=64)
            print("c1 layer", layer, "T", T, rep)


def _chain_layers(name, n, T_max, deterministic=False):
    w = synth.WORKLOADS[name]
    qs = [oracle.quantize_layer(synth.workload_layer(w, l)) for l in range(n)]
    return w, qs, [gu.make_gpu_layer(q, T_max, deterministic=deterministic) for q in qs]


@pytest.mark.parametrize("name,T", [("c0", 1), ("c0", 5), ("c0", 8), ("c1", 1), ("c1", 8), ("c0", 20)])
def test_forward_chain_matches_layer_by_layer(name, T):
    # mmoe_forward_chain: for up to 8 tokens one launch runs the whole stack (layer l + 1 reading layer
    # l's y rounded to BF16 inside the kernel); larger T runs one forward per layer.  Each layer's y
    # equals, bit for bit, that of its own forward on the BF16 rounding of the previous layer's y, and
    # matches the oracle on that input.  (Deterministic mode: y is added in the fixed order, so that it
    # is bit-reproducible on both the one-launch and the four-launch decode.)
    from moe_ffn_layer_fp32_b200.layer import MoELayer
    n = 4
    w, qs, Ls = _chain_layers(name, n, 64, deterministic=True)
    x0 = synth.draw_x(T, w.d, seed=500 + T)
    xd = gu.x_to_device(x0)
    ys = [torch.full((T, w.d), float("nan"), dtype=torch.float32, device="cuda") for _ in range(n)]
    MoELayer.forward_chain(Ls, xd, ys)
    torch.cuda.synchronize()
    xl = xd
    for l in range(n):
        y_ref = Ls[l].forward(xl)
        torch.cuda.synchronize()
        x_np = xl.view(torch.int16).cpu().numpy().view(np.uint16)
        y_or = oracle.moe_layer(qs[l], x_np)
        scale = np.abs(y_or).max()
        errs = (float(np.abs(ys[l].cpu().numpy() - y_or).max() / scale),
                float(np.abs(y_ref.cpu().numpy() - y_or).max() / scale))
        assert torch.equal(ys[l].view(torch.int32), y_ref.view(torch.int32)), (l, "chain / layer vs oracle", errs)
        rep = {}
        gu.check_y(ys[l].cpu().numpy(), y_or, rep)
        xl = y_ref.to(torch.bfloat16)
    # the same stack again: the launch left its counters ready for the next one
    ys2 = [torch.empty_like(y) for y in ys]
    MoELayer.forward_chain(Ls, xd, ys2)
    torch.cuda.synchronize()
    for a, b in zip(ys, ys2):
        assert torch.equal(a.view(torch.int32), b.view(torch.int32))
    for L in Ls:
        L.close()


@pytest.mark.parametrize("gating", [0, 2])
def test_forward_chain_with_router_bias(gating):
    # layers with a router bias (in the logit for gating 0, in the selection only for gating 2): the
    # stack in one launch equals the layers one by one
    from moe_ffn_layer_fp32_b200.layer import MoELayer
    w = synth.WORKLOADS["c0"]
    qs = [oracle.quantize_layer(synth.draw_layer(w.d, w.h, seed=70 + l, bias_coef=0.25), gating=gating)
          for l in range(3)]
    Ls = [gu.make_gpu_layer(q, 8, deterministic=True) for q in qs]
    T = 4
    xd = gu.x_to_device(synth.draw_x(T, w.d, seed=71))
    ys = [torch.empty((T, w.d), dtype=torch.float32, device="cuda") for _ in range(3)]
    MoELayer.forward_chain(Ls, xd, ys)
    torch.cuda.synchronize()
    xl = xd
    for l in range(3):
        y_ref = Ls[l].forward(xl)
        torch.cuda.synchronize()
        assert torch.equal(ys[l].view(torch.int32), y_ref.view(torch.int32)), l
        xl = y_ref.to(torch.bfloat16)
    for L in Ls:
        L.close()


@pytest.mark.parametrize("name,T", [("c0", 1), ("c0", 8), ("c1", 3), ("s2048", 2)])
def test_forward_chain_atomics_against_oracle(name, T):
    # the default chain (atomics into y): each layer's y matches the oracle on the BF16 rounding of the
    # previous layer's y from the same launch; a second launch agrees within FP32 rounding of the
    # summation order
    from moe_ffn_layer_fp32_b200.layer import MoELayer
    n = 5
    w, qs, Ls = _chain_layers(name, n, 8)
    xd = gu.x_to_device(synth.draw_x(T, w.d, seed=520 + T))
    ys = [torch.full((T, w.d), float("nan"), dtype=torch.float32, device="cuda") for _ in range(n)]
    MoELayer.forward_chain(Ls, xd, ys)
    torch.cuda.synchronize()
    xl = xd
    for l in range(n):
        x_np = xl.view(torch.int16).cpu().numpy().view(np.uint16)
        rep = {}
        gu.check_y(ys[l].cpu().numpy(), oracle.moe_layer(qs[l], x_np), rep)
        xl = ys[l].to(torch.bfloat16)
    ys2 = [torch.empty_like(y) for y in ys]
    MoELayer.forward_chain(Ls, xd, ys2)
    torch.cuda.synchronize()
    assert torch.max(torch.abs(ys2[0] - ys[0])) <= 1e-5 * torch.max(torch.abs(ys[0]))
    for L in Ls:
        L.close()


def test_forward_chain_rejects_mismatched_layers():
    from moe_ffn_layer_fp32_b200.layer import MoELayer
    w = synth.WORKLOADS["c0"]
    q = oracle.quantize_layer(synth.workload_layer(w))
    a = gu.make_gpu_layer(q, 8)
    b = MoELayer(w.d, 2 * w.h, max_tokens=8)  # another hidden size
    x = gu.x_to_device(synth.draw_x(2, w.d, seed=1))
    ys = [torch.empty((2, w.d), dtype=torch.float32, device="cuda") for _ in range(2)]
    with pytest.raises(_lib.MMoEError) as ei:
        MoELayer.forward_chain([a, b], x, ys)
    assert ei.value.status == 1  # INVALID_ARG
    a.close()
    b.close()


def test_c2_prefill():
    w, q = workload("c2")
    x = synth.workload_x(w)
    rep, out = _full_check(q, x, partial_rows=[0, 1, 4095, 8191, 8192, 10239])
    print("c2", rep)


def _sampled_check(name, n_sample=1024, T=None):
    # full-size workloads: routing, permutation and activation codes on every token, y on
    # n_sample seeded tokens (plus the first and the last), the INT32 partials of the first and
    # last row of every group that has rows (hot and cold groups alike)
    w, q = workload(name)
    T = w.T if T is None else T
    x = synth.workload_x(w, T=T)
    L = gu.make_gpu_layer(q, T)
    out = gu.run_gpu(L, q, x)
    rep = {}
    logits, probs, idx, gate = oracle.router(q, x)
    assert np.max(np.abs(out["logits"] - logits)) <= gu.LOGIT_TOL * max(1.0, np.abs(logits).max())
    gu.check_routing_and_permutation(q, out, idx, gate, probs, rep, logits)
    xq, sx = oracle.quantize_act(x)
    assert np.array_equal(out["xq"], xq) and np.array_equal(out["sx"], sx)
    rng = np.random.default_rng(7)
    toks = np.unique(np.concatenate([rng.choice(T, size=min(n_sample, T), replace=False), [0, T - 1]]))
    yref = oracle.moe_tokens(q, x, toks)
    gu.check_y(out["y"], yref, rep, rows=toks)
    rows = _group_edge_rows(out, q.E)
    rep["partial_rows"] = len(rows)
    gu.check_partials(L, q, out, rows)
    L.close()
    return rep, out


@pytest.mark.parametrize("name", ["c3a", "c3b"])
def test_c3_skewed_prefill(name):
    rep, out = _sampled_check(name)
    print(name, rep, "counts", out["counts"].tolist())
    if name == "c3a":
        assert (out["counts"][:60] == 0).sum() > 0, "the literal 1.5 bias leaves experts without tokens"


def test_c4_prefill_sampled():
    rep, out = _sampled_check("c4")
    print("c4", rep)


def test_c4_decode_batch64():
    w, q = workload("c4dec")
    x = synth.workload_x(w)
    rep, out = _full_check(q, x, partial_rows=[0, 63, 255, 256, 319])
    print("c4dec", rep)
