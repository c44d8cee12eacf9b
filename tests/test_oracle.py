"""Pins of the CPU oracle against facts that do not come from the oracle itself.

  * hand-derived Eq. (6) and activation-quantisation cases (tests/golden/);
  * exact-integer reductions where every group partial equals an int64 matmul;
  * the router against a float64 matmul and an independent top-k;
  * a dense numpy brute force over all 61 experts (float64 arithmetic);
  * invariants of Eq. (*): k distinct experts, counts, identical experts,
    k = E reducing to the full softmax mixture, E = k = 1 reducing to a dense FFN,
    closed forms for zero inputs.
"""
import numpy as np
import pytest

import oracle
from moe_ffn_layer_fp32_b200 import synth
from tests.conftest import read_cases


# ---------------------------------------------------------------------------
# independent helpers (numpy only; they share nothing with mmoe_oracle.c)
# ---------------------------------------------------------------------------
def codes_from_packed(p):
    p = np.asarray(p, dtype=np.uint8).astype(np.int64)
    out = np.zeros(p.shape[:-1] + (2 * p.shape[-1],), np.int64)
    for half, shift in ((0, 0), (1, 4)):
        v = (p >> shift) & 0xF
        out[..., half::2] = v - 16 * (v >= 8)
    return out


def bf16_to_f64(b):
    return synth.bf16_bits_to_f32(b).astype(np.float64)


def _expert_blocks(q, g):
    G, d = 32, q.d
    hid = q.h if g < q.E else q.hs
    wgu = codes_from_packed(q.w_gate_up[g * 2 * q.h * d // 2:][: 2 * hid * d // 2].reshape(2 * hid, d // 2))
    sgu = q.s_gate_up[g * 2 * q.h * d // G:][: 2 * hid * d // G].reshape(2 * hid, d // G).astype(np.float64)
    wd = codes_from_packed(q.w_down[g * d * q.h // 2:][: d * hid // 2].reshape(d, hid // 2))
    sd = q.s_down[g * d * q.h // G:][: d * hid // G].reshape(d, hid // G).astype(np.float64)
    return hid, wgu, sgu, wd, sd


def brute_force(q, x_bf16):
    """Dense float64 evaluation of Eq. (*) over all 61 experts, up to the SwiGLU output."""
    T, d, E, k = x_bf16.shape[0], q.d, q.E, q.k
    G = 32
    xf = bf16_to_f64(x_bf16)
    logits = (xf @ q.w_router.astype(np.float64)).astype(np.float32)
    if q.router_bias is not None:
        logits = (logits + q.router_bias).astype(np.float32)
    z = logits.astype(np.float64)
    p = np.exp(z - z.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    order = np.argsort(-logits, axis=1, kind="stable")[:, :k]
    # the activation codes are an integer decision: take it in FP32, like both implementations
    xf32 = xf.astype(np.float32)
    sx32 = (np.abs(xf32).max(axis=1) / np.float32(127.0)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        xq = np.where(sx32[:, None] > 0, np.clip(np.rint(xf32 / sx32[:, None]), -127, 127), 0).astype(np.int64)
    sx = sx32.astype(np.float64)
    acts = []
    for g in range(E + 1):
        hid, wgu, sgu, _, _ = _expert_blocks(q, g)
        P = np.einsum("tjc,njc->tnj", xq.reshape(T, d // G, G), wgu.reshape(2 * hid, d // G, G))
        gu = sx[:, None] * (P * sgu[None]).sum(axis=2)
        gv, uv = gu[:, :hid], gu[:, hid:]
        acts.append(gv / (1.0 + np.exp(-gv)) * uv)          # [T, hid]
    gate = p[np.arange(T)[:, None], order]
    return dict(logits=logits, probs=p, idx=order, gate=gate, xq=xq, sx=sx, acts=acts)


def brute_down(q, g, hq, sh):
    """Down projection of expert g in float64 from given INT8 codes hq[hid] and scale sh."""
    hid, _, _, wd, sd = _expert_blocks(q, g)
    Pd = (np.asarray(hq[:hid], np.int64).reshape(hid // 32, 32)[None] * wd.reshape(q.d, hid // 32, 32)).sum(-1)
    return sh * (Pd * sd).sum(axis=1)


def check_against_brute(q, x, y, D):
    """Compare an oracle run (y and its dumps) with the dense brute force.

    Integer stages (routing, x codes) must match exactly.  The SwiGLU requant is
    an FP32 decision in the oracle and a float64 one here, so an h code may
    differ by one only where a/s_h sits within 1e-3 of a rounding boundary;
    the down projection and the combine are then checked from the oracle's own
    codes, in float64.
    """
    bf = brute_force(q, x)
    T, k, E = x.shape[0], q.k, q.E
    assert np.array_equal(D["idx"], bf["idx"])
    assert np.array_equal(D["xq"].astype(np.int64), bf["xq"])
    assert np.array_equal(D["sx"], bf["sx"].astype(np.float32))
    assert np.max(np.abs(D["gate"] - bf["gate"])) < 1e-7
    yref = np.zeros((T, q.d))
    flips = total = 0
    for t in range(T):
        for s in range(k + 1):
            g = E if s == k else int(D["idx"][t, s])
            hid = q.h if g < E else q.hs
            a = bf["acts"][g][t]
            sh_ref = np.abs(a).max() / 127.0
            assert abs(D["sh"][t, s] - sh_ref) <= 1e-5 * sh_ref + 1e-30
            hq = D["hq"][t, s, :hid].astype(np.int64)
            if sh_ref > 0:
                r = a / sh_ref
                want = np.clip(np.rint(r), -127, 127)
                bad = hq != want
                near = np.abs(np.abs(r - np.floor(r)) - 0.5) < 1e-3
                assert np.all(np.abs(hq - want)[bad] == 1) and np.all(near[bad])
                flips += int(bad.sum())
            total += hid
            o = brute_down(q, g, hq, float(D["sh"][t, s]))
            assert np.max(np.abs(D["o"][t, s] - o)) <= 1e-5 * max(np.abs(o).max(), 1e-30)
            yref[t] += o if s == k else D["gate"][t, s] * o
    assert flips <= 0.01 * total
    assert np.max(np.abs(y - yref)) <= 1e-5 * np.abs(yref).max()
    return flips, total


# ---------------------------------------------------------------------------
# Eq. (6) and activation quantisation: hand-derived golden cases
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("case", read_cases("eq6_int4_cases.txt"), ids=lambda c: c["name"])
def test_eq6_golden(case):
    W = case["w"].astype(np.float32)[None, :]
    packed, scales = oracle.quantize_int4(W)
    assert scales[0, 0] == np.float32(case["s"][0])
    assert np.array_equal(codes_from_packed(packed)[0], case["q"].astype(np.int64))


@pytest.mark.parametrize("case", read_cases("act_int8_cases.txt"), ids=lambda c: c["name"])
def test_act_quant_golden(case):
    xb = synth.f32_to_bf16_bits(case["x"].astype(np.float32))[None, :]
    assert np.array_equal(synth.bf16_bits_to_f32(xb)[0], case["x"].astype(np.float32)), "fixture not BF16-exact"
    xq, sx = oracle.quantize_act(xb)
    assert sx[0] == np.float32(case["s"][0])
    assert np.array_equal(xq[0].astype(np.int64), case["q"].astype(np.int64))


def test_eq6_ranges_and_packing_random():
    rng = np.random.default_rng(5)
    W = (rng.standard_normal((37, 256)) * 0.02).astype(np.float32)
    W[3, 32:64] = 0.0
    packed, scales = oracle.quantize_int4(W)
    codes = codes_from_packed(packed)
    assert codes.min() >= -8 and codes.max() <= 7
    assert np.all(scales[3, 1] == 0) and np.all(codes[3, 32:64] == 0)
    # every group's largest |w| lands on +-7 or -8 (it is 7.5 s up to one rounding of s)
    g = np.abs(codes.reshape(37, 8, 32)).max(axis=2)
    nz = scales > 0
    assert np.all((g[nz] == 7) | (g[nz] == 8))
    # dequantised error is within half a step
    deq = codes.reshape(37, 8, 32) * scales[:, :, None].astype(np.float64)
    err = np.abs(deq - W.reshape(37, 8, 32).astype(np.float64))
    assert np.all(err <= 0.5 * scales[:, :, None] * (1 + 1e-6) + 1e-12)


def test_eq6_rejects_ragged_k():
    with pytest.raises(ValueError):
        oracle.quantize_int4(np.zeros((2, 48), np.float32))


# ---------------------------------------------------------------------------
# exact-integer reduction: group partials equal an int64 matmul
# ---------------------------------------------------------------------------
def _exact_weights(rng, rows, K, e):
    """FP32 weights whose Eq. (6) scale is exactly 2^e and whose codes are known."""
    s = np.float32(2.0 ** e)
    codes = rng.integers(-7, 8, size=(rows, K)).astype(np.int64)
    g = K // 32
    pos = rng.integers(0, 32, size=(rows, g))
    sign = rng.integers(0, 2, size=(rows, g))
    W = codes.astype(np.float32) * s
    for r in range(rows):
        for j in range(g):
            c = j * 32 + pos[r, j]
            W[r, c] = np.float32(7.5) * s if sign[r, j] else np.float32(-7.5) * s
            codes[r, c] = 7 if sign[r, j] else -8
    return W, codes


def test_partials_equal_int64_matmul():
    rng = np.random.default_rng(11)
    d, h, E, T = 64, 64, 60, 9
    lw = synth.LayerWeights(d=d, h=h, hs=h, E=E, w_router=(rng.standard_normal((d, E)) * 0.02).astype(np.float32),
                            router_bias=None)
    codes_gu, codes_d = [], []
    for g in range(E + 1):
        Wgu, cgu = _exact_weights(rng, 2 * h, d, -5)
        Wd, cd = _exact_weights(rng, d, h, -6)
        lw.w_gate_up.append(Wgu); lw.w_down.append(Wd)
        codes_gu.append(cgu); codes_d.append(cd)
    q = oracle.quantize_layer(lw)
    # Eq. (6) gives back exactly the planted codes and scales
    for g in (0, 17, 60):
        cgu, sgu, cd, sd = q.expert_codes(g)
        assert np.array_equal(cgu.astype(np.int64), codes_gu[g])
        assert np.all(sgu == np.float32(2.0 ** -5)) and np.all(sd == np.float32(2.0 ** -6))
    # integer activations with +-127 in every row: s_x = 1 and x_q = x
    xi = rng.integers(-127, 128, size=(T, d))
    xi[:, 0] = np.where(rng.integers(0, 2, T) == 1, 127, -127)
    x = synth.f32_to_bf16_bits(xi.astype(np.float32))
    y, D = oracle.moe_layer(q, x, dumps=True, partials=True)
    assert np.all(D["sx"] == 1.0)
    assert np.array_equal(D["xq"].astype(np.int64), xi)
    for t in range(T):
        for s in range(q.k + 1):
            g = q.E if s == q.k else D["idx"][t, s]
            Pg = (xi[t].reshape(d // 32, 32)[None] * codes_gu[g][:h].reshape(h, d // 32, 32)).sum(-1)
            Pu = (xi[t].reshape(d // 32, 32)[None] * codes_gu[g][h:].reshape(h, d // 32, 32)).sum(-1)
            assert np.array_equal(D["pg"][t, s], Pg)
            assert np.array_equal(D["pu"][t, s], Pu)
            hq = D["hq"][t, s].astype(np.int64)
            Pd = (hq.reshape(h // 32, 32)[None] * codes_d[g].reshape(d, h // 32, 32)).sum(-1)
            assert np.array_equal(D["pd"][t, s], Pd)


# ---------------------------------------------------------------------------
# router
# ---------------------------------------------------------------------------
def test_router_against_float64_and_stable_topk(c0_layer, c0_oracle):
    w, lw, q, x = c0_layer
    y, D = c0_oracle
    ref = bf16_to_f64(x) @ q.w_router.astype(np.float64)
    assert np.max(np.abs(D["logits"] - ref)) < 1e-5
    assert np.allclose(D["probs"].sum(axis=1), 1.0, atol=1e-6)
    order = np.argsort(-D["logits"], axis=1, kind="stable")[:, :4]
    assert np.array_equal(D["idx"], order)
    assert np.array_equal(D["gate"], np.take_along_axis(D["probs"], D["idx"], axis=1))


def test_router_ties_lowest_index_first():
    d, E = 64, 60
    wr = np.zeros((d, E), np.float32)
    wr[:, 7] = 0.01
    wr[:, 3] = 0.01
    wr[:, 50] = 0.01
    wr[:, 9] = 0.005
    wr[:, 2] = 0.005
    lw = synth.LayerWeights(d=d, h=32, hs=32, E=E, w_router=wr, router_bias=None)
    for g in range(E + 1):
        lw.w_gate_up.append(np.zeros((64, d), np.float32))
        lw.w_down.append(np.zeros((d, 32), np.float32))
    q = oracle.quantize_layer(lw)
    x = synth.f32_to_bf16_bits(np.ones((2, d), np.float32))
    _, _, idx, gate = oracle.router(q, x)
    assert idx.tolist() == [[3, 7, 50, 2], [3, 7, 50, 2]]
    assert gate[0, 0] == gate[0, 1] == gate[0, 2]


def test_router_bias_shifts_selection():
    w = synth.WORKLOADS["c0"]
    lw = synth.draw_layer(w.d, w.h, seed=3, bias_coef=1.5)
    q = oracle.quantize_layer(lw)
    x = synth.draw_x(128, w.d, seed=4)
    logits, probs, idx, gate = oracle.router(q, x)
    hot = int(np.argmax(lw.router_bias))            # rank 0: bias 0, every other bias < 0
    assert lw.router_bias[hot] == 0.0
    assert np.mean(np.any(idx == hot, axis=1)) > 0.9
    nob = bf16_to_f64(x) @ q.w_router.astype(np.float64)
    assert np.max(np.abs(logits - (nob.astype(np.float32) + lw.router_bias))) < 1e-5


def test_sigmoid_gating_normalised():
    w = synth.WORKLOADS["c0"]
    lw = synth.workload_layer(w)
    q = oracle.quantize_layer(lw, gating=1)
    x = synth.workload_x(w)
    logits, probs, idx, gate = oracle.router(q, x)
    assert np.allclose(gate.sum(axis=1), 1.0, atol=1e-6)
    assert np.allclose(probs, 1 / (1 + np.exp(-logits.astype(np.float64))), atol=1e-7)
    q0 = oracle.quantize_layer(lw, gating=0)
    assert np.array_equal(oracle.router(q0, x)[2], idx), "selection is the same for any monotone gate"


def _sel_bias_routing_ref(q, x):
    """Selection-only bias routing (gating 2) from an independent float64 matmul: logits without
    the bias, p = sigmoid, key = FP32(p + b), stable top-k of the key, gates = p / sum over the
    selected.  Returns (logits32, probs32, key32, idx, gate)."""
    l64 = bf16_to_f64(x) @ q.w_router.astype(np.float64)
    l32 = l64.astype(np.float32)
    p32 = (1.0 / (1.0 + np.exp(-l32.astype(np.float64)))).astype(np.float32)
    key = (p32 + q.router_bias.astype(np.float32)).astype(np.float32)
    idx = np.argsort(-key, axis=1, kind="stable")[:, :q.k]
    sel = np.take_along_axis(p32.astype(np.float64), idx, axis=1)
    return l32, p32, key, idx, sel / sel.sum(axis=1, keepdims=True)


def test_selection_bias_moves_selection_not_gates():
    # gating 2 (auxiliary-loss-free balancing): the per-expert bias joins the sigmoid score only to
    # pick the top-k; the reported logits exclude it and the gates are the unbiased scores,
    # normalised over the selected experts
    w = synth.WORKLOADS["c0"]
    lw = synth.draw_layer(w.d, w.h, seed=5, bias_coef=0.25)
    q = oracle.quantize_layer(lw, gating=2)
    x = synth.draw_x(256, w.d, seed=6)
    logits, probs, idx, gate = oracle.router(q, x)
    l32, p32, key, idx_ref, gate_ref = _sel_bias_routing_ref(q, x)
    assert np.max(np.abs(logits - l32)) < 1e-5                 # no bias in the logits
    assert np.allclose(probs, p32, atol=1e-7)
    # the oracle's selection from its own scores: the top-k of p + b (exact), lower index first on ties
    own_key = (probs + lw.router_bias.astype(np.float32)).astype(np.float32)
    assert np.array_equal(idx, np.argsort(-own_key, axis=1, kind="stable")[:, :q.k])
    srt = -np.sort(-key, axis=1)
    clear = srt[:, q.k - 1] - srt[:, q.k] > 1e-5               # away from the selection margin
    assert clear.mean() > 0.9
    assert np.array_equal(idx[clear], idx_ref[clear])
    assert np.allclose(gate.sum(axis=1), 1.0, atol=1e-6)
    assert np.max(np.abs(gate[clear] - gate_ref[clear])) < 1e-6
    # the bias really moves the selection: without it the top-k differs on most tokens
    q1 = oracle.quantize_layer(synth.LayerWeights(d=lw.d, h=lw.h, hs=lw.hs, E=lw.E, w_router=lw.w_router,
                                                  router_bias=None, w_gate_up=lw.w_gate_up, w_down=lw.w_down),
                               gating=1)
    idx1 = oracle.router(q1, x)[2]
    assert np.mean(np.any(np.sort(idx1, axis=1) != np.sort(idx, axis=1), axis=1)) > 0.5


def test_selection_bias_zero_equals_sigmoid_gating():
    # with a zero bias the key is the sigmoid score, a monotone function of the logit: the same
    # experts and gates as gating 1 (no two scores of these tokens round to the same FP32 value)
    w = synth.WORKLOADS["c0"]
    lw = synth.workload_layer(w)
    lw0 = synth.LayerWeights(d=lw.d, h=lw.h, hs=lw.hs, E=lw.E, w_router=lw.w_router,
                             router_bias=np.zeros(lw.E, np.float32), w_gate_up=lw.w_gate_up, w_down=lw.w_down)
    x = synth.workload_x(w)
    _, p2, i2, g2 = oracle.router(oracle.quantize_layer(lw0, gating=2), x)
    _, _, i1, g1 = oracle.router(oracle.quantize_layer(lw, gating=1), x)
    assert all(len(set(r.tolist())) == len(r) for r in p2)
    assert np.array_equal(i1, i2) and np.array_equal(g1, g2)


def test_selection_bias_layer_brute_force():
    # the whole layer with gating 2 against the dense float64 brute force, routed by the
    # independent reference above
    w = synth.WORKLOADS["c0"]
    lw = synth.draw_layer(w.d, w.h, seed=7, bias_coef=1.5)
    q = oracle.quantize_layer(lw, gating=2)
    x = synth.draw_x(32, w.d, seed=8)
    y, D = oracle.moe_layer(q, x, dumps=True)
    _, _, key, idx_ref, gate_ref = _sel_bias_routing_ref(q, x)
    srt = -np.sort(-key, axis=1)
    assert np.all(srt[:, q.k - 1] - srt[:, q.k] > 1e-6)
    assert np.array_equal(D["idx"], idx_ref)
    assert np.max(np.abs(D["gate"] - gate_ref)) < 1e-6
    # the expert side (SwiGLU codes, down projection) is pinned by the brute-force test of gating 0;
    # here the layer is recombined from the oracle's own codes with the reference routing and gates
    yref = np.zeros((x.shape[0], q.d))
    for t in range(x.shape[0]):
        for s in range(q.k + 1):
            g = q.E if s == q.k else int(idx_ref[t, s])
            o = brute_down(q, g, D["hq"][t, s], float(D["sh"][t, s]))
            yref[t] += o if s == q.k else gate_ref[t, s] * o
    assert np.max(np.abs(y - yref)) <= 1e-5 * np.abs(yref).max()


# ---------------------------------------------------------------------------
# brute force over all experts
# ---------------------------------------------------------------------------
def test_brute_force_c0(c0_layer, c0_oracle):
    w, lw, q, x = c0_layer
    y, D = c0_oracle
    check_against_brute(q, x, y, D)


# ---------------------------------------------------------------------------
# invariants of Eq. (*)
# ---------------------------------------------------------------------------
def test_k_distinct_experts_and_counts(c0_layer, c0_oracle):
    w, lw, q, x = c0_layer
    y, D = c0_oracle
    idx = D["idx"]
    assert all(len(set(r)) == 4 for r in idx.tolist())
    assert idx.min() >= 0 and idx.max() < 60
    cnt = np.bincount(idx.ravel(), minlength=60)
    assert cnt.sum() == 4 * w.T
    assert np.all(D["gate"].sum(axis=1) <= 1.0 + 1e-6)
    assert np.all(np.diff(D["gate"], axis=1) <= 0), "gates follow the logit order"


def _identical_expert_layer(w, seed=21):
    lw = synth.draw_layer(w.d, w.h, seed=seed)
    for g in range(1, lw.E):
        lw.w_gate_up[g] = lw.w_gate_up[0]
        lw.w_down[g] = lw.w_down[0]
    return lw


def _ffn(q, g, xq_row, sx):
    hq, sh = oracle.expert_gate_up(q, g, xq_row, sx)
    return oracle.expert_down(q, g, hq, sh).astype(np.float64)


def test_identical_experts_reduce_to_dense(c0_layer):
    w = c0_layer[0]
    q = oracle.quantize_layer(_identical_expert_layer(w))
    x = synth.draw_x(16, w.d, seed=22)
    y, D = oracle.moe_layer(q, x, dumps=True)
    for t in range(16):
        f = _ffn(q, 0, D["xq"][t], D["sx"][t])
        fs = _ffn(q, q.E, D["xq"][t], D["sx"][t])
        ref = D["gate"][t].astype(np.float64).sum() * f + fs
        assert np.max(np.abs(y[t] - ref)) <= 1e-5 * max(np.abs(ref).max(), 1e-30)


def test_k_equals_E_is_full_softmax_mixture(c0_layer):
    w = c0_layer[0]
    lw = synth.draw_layer(w.d, w.h, seed=23)
    q = oracle.quantize_layer(lw, k=60)
    x = synth.draw_x(4, w.d, seed=24)
    y, D = oracle.moe_layer(q, x, dumps=True)
    for t in range(4):
        assert sorted(D["idx"][t].tolist()) == list(range(60))
        ref = _ffn(q, q.E, D["xq"][t], D["sx"][t])
        for e in range(60):
            ref = ref + D["probs"][t, e].astype(np.float64) * _ffn(q, e, D["xq"][t], D["sx"][t])
        assert np.max(np.abs(y[t] - ref)) <= 1e-5 * np.abs(ref).max()
    # with identical experts as well: y = FFN(x) + FFN_s(x)
    q2 = oracle.quantize_layer(_identical_expert_layer(w, seed=25), k=60)
    y2, D2 = oracle.moe_layer(q2, x, dumps=True)
    for t in range(4):
        ref = _ffn(q2, 0, D2["xq"][t], D2["sx"][t]) + _ffn(q2, q2.E, D2["xq"][t], D2["sx"][t])
        assert np.max(np.abs(y2[t] - ref)) <= 1e-5 * np.abs(ref).max()


def test_single_expert_top1_is_dense_swiglu_plus_shared(c0_layer):
    w = c0_layer[0]
    lw = synth.draw_layer(w.d, w.h, E=1, seed=26)
    q = oracle.quantize_layer(lw, k=1)
    x = synth.draw_x(8, w.d, seed=27)
    y, D = oracle.moe_layer(q, x, dumps=True)
    assert np.all(D["gate"] == 1.0) and np.all(D["idx"] == 0)
    check_against_brute(q, x, y, D)


def test_zero_inputs_closed_forms(c0_layer):
    w, lw, q, x = c0_layer
    z = np.zeros((3, w.d), np.uint16)
    y, D = oracle.moe_layer(q, z, dumps=True)
    assert np.all(D["sx"] == 0) and np.all(D["xq"] == 0)
    assert np.all(y == 0)
    # zero gate projections: silu(0) * u = 0, so every expert output is 0
    lz = synth.draw_layer(w.d, w.h, seed=28)
    for g in range(lz.E + 1):
        lz.w_gate_up[g][: w.h] = 0.0
    qz = oracle.quantize_layer(lz)
    y2, D2 = oracle.moe_layer(qz, x[:5], dumps=True)
    assert np.all(D2["sh"] == 0) and np.all(D2["hq"] == 0) and np.all(y2 == 0)


def test_tokens_subset_matches_full(c0_layer, c0_oracle):
    w, lw, q, x = c0_layer
    y, _ = c0_oracle
    toks = np.array([63, 0, 17, 17, 40])
    assert np.array_equal(oracle.moe_tokens(q, x, toks), y[toks])
