"""Helpers for the GPU parity tests: run the library through its C ABI and
compare every stage with the CPU oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from moe_ffn_layer_fp32_b200 import _lib, build, synth

MARGIN = 1e-5      # router margin p_(k) - p_(k+1) under which a token's routing is not required to match
Y_TOL = 2e-3       # max|dy| <= Y_TOL * max|y_ref|
LOGIT_TOL = 1e-5   # |l_gpu - l_ref| <= LOGIT_TOL * max(1, max|l_ref|): FP32 sums against the oracle's FP64 sums
GATE_RTOL = 1e-6   # rounding of exp and of the division in one gate


def ensure_built():
    build.build()


def x_to_device(x_np: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x_np).view(np.int16)).cuda().view(torch.bfloat16)


def make_gpu_layer(q: oracle.QuantizedLayer, max_tokens: int, deterministic: bool = False, cuda_cores: bool = False,
                   decode: bool = True, atomic_combine: bool = False, tc_int8: bool = False,
                   fused_decode: bool = True, fused_requant: bool = False):
    from moe_ffn_layer_fp32_b200.layer import MoELayer
    L = MoELayer(q.d, q.h, shared_hidden=q.hs, n_experts=q.E, top_k=q.k, max_tokens=max_tokens,
                 gating=q.gating, has_router_bias=q.router_bias is not None, deterministic=deterministic,
                 cuda_cores=cuda_cores, decode=decode, atomic_combine=atomic_combine, tc_int8=tc_int8,
                 fused_decode=fused_decode, fused_requant=fused_requant)
    L.load(q.w_router, q.router_bias, q.w_gate_up, q.s_gate_up, q.w_down, q.s_down)
    return L


def run_gpu(L, q, x_np, stages=True):
    T = x_np.shape[0]
    x = x_to_device(x_np)
    dev = x.device
    idx = torch.full((max(T, 1), q.k), -1, dtype=torch.int32, device=dev)
    gate = torch.zeros((max(T, 1), q.k), dtype=torch.float32, device=dev)
    cnt = torch.zeros(q.E + 1, dtype=torch.int32, device=dev)
    y = L.forward(x, topk_idx=idx, topk_gate=gate, expert_counts=cnt)
    torch.cuda.synchronize()
    out = dict(y=y.cpu().numpy(), idx=idx[:T].cpu().numpy(), gate=gate[:T].cpu().numpy(), counts=cnt.cpu().numpy())
    if stages and T > 0:
        R, hm = T * (q.k + 1), max(q.h, q.hs)
        out["xq"] = L.stage(_lib.STAGE_XQ, (T, q.d), torch.int8).cpu().numpy()
        out["sx"] = L.stage(_lib.STAGE_SX, (T,), torch.float32).cpu().numpy()
        out["offsets"] = L.stage(_lib.STAGE_OFFSETS, (q.E + 2,), torch.int32).cpu().numpy()
        out["row_src"] = L.stage(_lib.STAGE_ROW_SRC, (R,), torch.int32).cpu().numpy()
        out["slot_row"] = L.stage(_lib.STAGE_SLOT_ROW, (T, q.k), torch.int32).cpu().numpy()
        out["hq"] = L.stage(_lib.STAGE_HQ, (R, hm), torch.int8).cpu().numpy()
        out["sh"] = L.stage(_lib.STAGE_SH, (R,), torch.float32).cpu().numpy()
        out["logits"] = L.stage(_lib.STAGE_LOGITS, (T, q.E), torch.float32).cpu().numpy()
        torch.cuda.synchronize()
    return out


def selection_keys(q, probs: np.ndarray, logits: np.ndarray) -> np.ndarray:
    """What the top-k is taken over: the logits (gating 0, 1), the biased sigmoid scores (gating 2)."""
    if q.gating == 2:
        b = np.zeros(q.E, np.float32) if q.router_bias is None else q.router_bias
        return (probs + b).astype(np.float32)
    return logits


def router_margin(probs: np.ndarray, k: int) -> np.ndarray:
    if probs.shape[1] <= k:
        return np.full(probs.shape[0], np.inf)
    s = -np.sort(-probs, axis=1)
    return s[:, k - 1] - s[:, k]


def group_of_rows(offsets: np.ndarray, E: int) -> np.ndarray:
    R = offsets[E + 1]
    g = np.zeros(R, np.int64)
    for e in range(E + 1):
        g[offsets[e]:offsets[e + 1]] = e
    return g


def check_routing_and_permutation(q, out, ref_idx, ref_gate, ref_probs, report, ref_logits=None):
    """Routing bit-exact outside the margin band; permutation valid and stable.

    Margin: tokens whose k-th and (k+1)-th softmax probabilities (gating 0, 1) or
    biased sigmoid scores (gating 2) differ by less than MARGIN may select
    differently and are counted, not compared.

    Gates: the GPU's logits are FP32 sums of d exact products, the oracle's FP64
    sums rounded once, and the logit check bounds their difference by
    LOGIT_TOL * max(1, max|l_ref|).  A softmax gate exp(l_e - m) / sum exp(l - m),
    and a top-k-normalised sigmoid score alike, moves by at most about twice the
    largest logit difference in relative terms, so the fixed bound per workload is
    2 LOGIT_TOL max(1, max|l_ref|) + GATE_RTOL."""
    T, k, E = out["idx"].shape[0], q.k, q.E
    if ref_logits is None:
        ref_logits = np.zeros((T, E), np.float32)
    if q.gating == 2:
        keys = selection_keys(q, ref_probs, ref_logits)
        s_ = -np.sort(-keys, axis=1)
        margin = s_[:, k - 1] - s_[:, k] if E > k else np.full(T, np.inf)
    else:
        margin = router_margin(ref_probs, k)
    excl = margin < MARGIN
    report["margin_excluded"] = int(excl.sum())
    ok = ~excl
    assert np.array_equal(out["idx"][ok], ref_idx[ok]), "routing differs on tokens outside the margin band"
    g, rg = out["gate"][ok].astype(np.float64), ref_gate[ok].astype(np.float64)
    bound = 2.0 * LOGIT_TOL * max(1.0, float(np.abs(ref_logits).max()) if ref_logits.size else 1.0) + GATE_RTOL
    if "logits" in out:
        dl = np.abs(out["logits"].astype(np.float64) - ref_logits.astype(np.float64)).max() if T else 0.0
        report["logit_max_abs_err"] = float(dl)
    rel = np.abs(g - rg) / np.maximum(np.abs(rg), 1e-30)
    report["gate_max_rel_err"] = float(rel.max()) if rel.size else 0.0
    report["gate_bound"] = bound
    assert np.all(rel <= bound), (rel.max(), bound)
    idx = out["idx"]
    assert np.all((idx >= 0) & (idx < E))
    assert all(len(set(r)) == k for r in idx.tolist())
    cnt = np.bincount(idx.ravel(), minlength=E)
    assert np.array_equal(out["counts"][:E], cnt) and out["counts"][E] == T
    if "offsets" not in out:
        return
    off = out["offsets"]
    assert off[0] == 0 and np.array_equal(np.diff(off[: E + 1]), cnt) and off[E] == T * k and off[E + 1] == T * (k + 1)
    rs, sr = out["row_src"], out["slot_row"]
    # slot -> row -> token is the identity and rows fall in their expert's range
    for t in range(T):
        for j in range(k):
            r = sr[t, j]
            assert rs[r] == t and off[idx[t, j]] <= r < off[idx[t, j] + 1]
    # stable: within an expert, (token, slot) ascending
    slot_of_row = np.empty(T * k, np.int64)
    slot_of_row[sr.ravel()] = np.arange(T * k)
    for e in range(E):
        s = slot_of_row[off[e]:off[e + 1]]
        assert np.all(np.diff(s) > 0)
    assert np.array_equal(rs[T * k:], np.arange(T))


def check_hq(q, out, ref_dumps, report, tokens=None):
    """SwiGLU output codes: equal, or one apart (FP32 summation / expf ulps near a rounding boundary)."""
    T, k = out["idx"].shape[0], q.k
    tokens = range(T) if tokens is None else tokens
    mism = total = 0
    for t in tokens:
        for s in range(k + 1):
            if s < k and out["idx"][t, s] != ref_dumps["idx"][t, s]:
                continue
            r = out["slot_row"][t, s] if s < k else T * k + t
            g = out["idx"][t, s] if s < k else q.E
            hid = q.h if g < q.E else q.hs
            a = out["hq"][r, :hid].astype(np.int64)
            b = ref_dumps["hq"][t, s, :hid].astype(np.int64)
            assert np.all(np.abs(a - b) <= 1)
            mism += int((a != b).sum())
            total += hid
            sh_r = ref_dumps["sh"][t, s]
            assert abs(out["sh"][r] - sh_r) <= 1e-5 * abs(sh_r) + 1e-30
    report["hq_mismatch"] = mism
    report["hq_total"] = total
    assert mism <= max(2, 2e-3 * total), (mism, total)


def check_y(y, yref, report, rows=None):
    if rows is not None:
        y = y[rows]
    scale = np.abs(yref).max()
    err = np.abs(y.astype(np.float64) - yref.astype(np.float64)).max() if y.size else 0.0
    report["y_max_abs_err"] = float(err)
    report["y_rel_err"] = float(err / scale) if scale > 0 else float(err)
    assert err <= Y_TOL * scale + 1e-30, (err, scale)


def check_partials(L, q, out, rows):
    """INT32 group partials of the GPU GEMMs equal the oracle's, bit for bit (down: from the GPU's h codes)."""
    off, rs = out["offsets"], out["row_src"]
    grp = group_of_rows(off, q.E)
    rows = np.asarray(rows)
    for r0 in rows:
        r0 = int(r0)
        pgu = L.partials(0, r0, 1).cpu().numpy()[0]
        pd = L.partials(1, r0, 1).cpu().numpy()[0]
        g = int(grp[r0])
        t = int(rs[r0])
        hid = q.h if g < q.E else q.hs
        hq, sh, rpg, rpu = oracle.expert_gate_up(q, g, out["xq"][t], out["sx"][t], partials=True)
        assert np.array_equal(pgu[:hid], rpg), f"gate partials of row {r0}"
        hm = max(q.h, q.hs)
        assert np.array_equal(pgu[hm:hm + hid], rpu), f"up partials of row {r0}"
        _, rpd = oracle.expert_down(q, g, out["hq"][r0], float(out["sh"][r0]), partials=True)
        assert np.array_equal(pd[:, : hid // 32], rpd), f"down partials of row {r0}"
