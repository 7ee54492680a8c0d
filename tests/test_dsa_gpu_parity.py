"""GPU parity of the sparse-attention key selection: the CUDA path (through the
C ABI) against the CPU oracle on seeded inputs.

Rules (the oracle computes in double from the same bf16 / fp32 inputs):
  * scores: every visible entry within the rounding bound of fp32 arithmetic,
        |S_gpu - S_oracle| <= 2 * (D + NH + 4) * 2^-24 * sum_h |w_h| sum_d |q_hd k_d| / sqrt(NH*D)
    (D products summed per head, NH weighted terms, one scale: each fp32 add
    contributes at most one unit roundoff of the running magnitude; the factor
    2 covers an accumulator that truncates instead of rounding);
  * the top-k is an integer decision, so it is checked in the precision the
    kernel takes it: the GPU's selection must equal the oracle's selection
    applied to the GPU's own fp32 scores, exactly;
  * against the oracle's selection from its double scores the sets must be
    equal on every row whose gap between the k-th and (k+1)-th oracle score
    exceeds twice that row's score bound (several selections are correct
    inside a near tie); near-tie rows are counted and their disagreements
    must lie inside the tie band.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from sigmoid_routed_mixture_b200 import dsa
from sigmoid_routed_mixture_b200 import workloads as W

pytestmark = pytest.mark.gpu


def dev_bf16(bits):
    return torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)


def score_bound(q, k, w, rows):
    """Per-entry bound for the listed (b, t) rows: [n, S]."""
    B, T, NH, D = q.shape
    qa = np.abs(W.bf16_bits_to_f32(q).astype(np.float64))
    ka = np.abs(W.bf16_bits_to_f32(k).astype(np.float64))
    wa = np.abs(w.astype(np.float64))
    out = []
    for b, t in rows:
        m = wa[b, t] @ (qa[b, t] @ ka[b].T)  # sum_h |w_h| sum_d |q_hd k_d|
        out.append(2.0 * (D + NH + 4) * 2.0 ** -24 * m / np.sqrt(NH * D))
    return np.array(out)


class Run:
    def __init__(self, wl: W.DsaWorkload):
        self.wl = wl
        self.q, self.k, self.w = W.dsa_inputs(wl)
        self.cfg = dsa.Config(wl.B, wl.T, wl.S, wl.n_heads, wl.head_dim, wl.topk)
        self.ws = dsa.workspace(self.cfg)
        qd, kd, wd = dev_bf16(self.q), dev_bf16(self.k), torch.from_numpy(self.w).cuda()
        self.scores_dev = torch.full((wl.B, wl.T, wl.S), float("-inf"), dtype=torch.float32,
                                     device="cuda")
        self.sel = dsa.select(self.cfg, qd, kd, wd, self.ws, scores_out=self.scores_dev)
        torch.cuda.synchronize()
        self.sel = self.sel.cpu().numpy()
        self.scores = self.scores_dev.cpu().numpy()
        self.dev = (qd, kd, wd)

    def device_error(self):
        from sigmoid_routed_mixture_b200 import moe
        return moe.device_error(self.ws)

    def check_rows(self, rows):
        wl = self.wl
        n_sel = min(wl.topk, wl.S)
        bs = sorted({b for b, _ in rows})
        near = 0
        for b in bs:
            ts = [t for bb, t in rows if bb == b]
            o = O.dsa_scores(self.q[b:b + 1], self.k[b:b + 1], self.w[b:b + 1])[0][ts]
            bound = score_bound(self.q, self.k, self.w, [(b, t) for t in ts])
            for i, t in enumerate(ts):
                pos = wl.S - wl.T + t
                g = self.scores[b, t, :pos + 1].astype(np.float64)
                ref = o[i, :pos + 1]
                assert np.all(np.isfinite(ref)) and not np.isfinite(o[i, pos + 1:]).any()
                err = np.abs(g - ref)
                assert np.all(err <= bound[i, :pos + 1]), (b, t, float(err.max()))
                # exact: the kernel's top-k on its own scores
                gs = np.full(wl.S, -np.inf)
                gs[:pos + 1] = g
                own, _, _ = O.dsa_select(gs, wl.topk)
                assert np.array_equal(self.sel[b, t], own), (b, t)
                # against the oracle's selection: equal unless inside a near tie
                full = np.full(wl.S, -np.inf)
                full[:pos + 1] = ref
                osel, kth, nxt = O.dsa_select(full, wl.topk)
                band = 2.0 * bound[i, :pos + 1].max()
                if not np.isfinite(kth) or kth - nxt > band:  # every visible key taken, or no tie
                    assert np.array_equal(self.sel[b, t], osel), (b, t)
                else:
                    near += 1
                    diff = set(self.sel[b, t].tolist()) ^ set(osel.tolist())
                    for s in diff:
                        assert abs(full[s] - kth) <= band, (b, t, s)
                assert len(self.sel[b, t]) == n_sel
                assert np.all(np.diff(self.sel[b, t]) > 0)
        return near


def all_rows(wl):
    return [(b, t) for b in range(wl.B) for t in range(wl.T)]


def test_tiny_full_parity():
    wl = W.DSA_WORKLOADS["dsa_tiny"]
    r = Run(wl)
    assert r.device_error() == 0
    r.check_rows(all_rows(wl))


@pytest.mark.parametrize("B,T,S,topk", [(3, 37, 300, 50), (1, 5, 1000, 128), (2, 129, 129, 40),
                                        (1, 1, 777, 700), (2, 333, 333, 100), (3, 250, 700, 300)])
def test_ragged_queries_keys_and_cache(B, T, S, topk):
    """Query counts not a multiple of the 8-query block, key counts not a multiple
    of the 128-key tile, and a cache (T < S: queries sit at the last T positions);
    enough rows for the persistent top-k, with rows that do (S % 4 == 0) and do
    not start on 16-byte boundaries."""
    wl = W.DsaWorkload("ragged", B=B, T=T, S=S, topk=topk, seed=2100 + T + S)
    r = Run(wl)
    assert r.device_error() == 0
    r.check_rows(all_rows(wl))


@pytest.mark.parametrize("NH,D", [(64, 128), (128, 128), (32, 64), (128, 64)])
def test_head_shapes(NH, D):
    wl = W.DsaWorkload("heads", B=2, T=70, S=260, n_heads=NH, head_dim=D, topk=33,
                       seed=2200 + NH + D)
    r = Run(wl)
    assert r.device_error() == 0
    r.check_rows(all_rows(wl))


@pytest.mark.parametrize("NH,D", [(32, 128), (64, 64), (128, 128)])
def test_single_query_sequences(NH, D):
    """One query per sequence (decode): tiles of one query's heads (N = NH)."""
    wl = W.DsaWorkload("decode", B=5, T=1, S=3000, n_heads=NH, head_dim=D, topk=300,
                       seed=2250 + NH + D)
    r = Run(wl)
    assert r.device_error() == 0
    r.check_rows(all_rows(wl))


def test_short_prompt_lists_every_key():
    """S <= topk: every query selects keys 0 .. S-1 (the page's short-prompt rule)."""
    wl = W.DsaWorkload("short", B=2, T=200, S=200, topk=2048, seed=2300)
    r = Run(wl)
    assert r.sel.shape == (2, 200, 200)
    assert all(np.array_equal(r.sel[b, t], np.arange(200)) for b in range(2) for t in range(200))


def test_exact_ties_go_to_the_lower_key():
    """Duplicated key rows give bit-identical scores.  With an odd topk exactly one
    pair is split at the threshold, and the lower index of that pair must win."""
    wl = W.DsaWorkload("ties", B=1, T=1, S=600, topk=101, seed=2400)
    q, k, w = W.dsa_inputs(wl)
    k = k.copy()
    k[0, 300:600] = k[0, 0:300]  # key s + 300 repeats key s
    cfg = dsa.Config(1, 1, 600, topk=101)
    ws = dsa.workspace(cfg)
    sel = dsa.select(cfg, dev_bf16(q), dev_bf16(k), torch.from_numpy(w).cuda(), ws).cpu().numpy()
    chosen = set(sel[0, 0].tolist())
    split = [s for s in range(300) if (s in chosen) != (s + 300 in chosen)]
    assert len(split) == 1 and split[0] in chosen
    osel, _, _ = O.dsa_select(O.dsa_scores(q, k, w), 101)
    assert np.array_equal(sel, osel)


def test_topk_alone_on_given_scores_is_exact():
    """dsa_topk on fp32 scores chosen by the test equals the oracle's order on the
    same values (with planted ties and a causal tail that must be ignored)."""
    B, T, S, topk = 2, 6, 5000, 2048
    rng = np.random.default_rng(5)
    sc = rng.standard_normal((B, T, S)).astype(np.float32)
    vis = sc[0, 5, :S - T + 5 + 1]
    thr = np.sort(vis)[-topk]                  # the row's topk-th score
    sc[0, 5, 100:140] = thr                    # a run of 40 equal scores at the threshold
    sc[1, :, :] = np.round(sc[1] * 4) / 4      # many ties everywhere
    sc[1, 2, ::3] = -0.0                       # signed zeros: -0 and +0 are equal scores
    sc[1, 2, 1::3] = 0.0
    cfg = dsa.Config(B, T, S, topk=topk)
    ws = dsa.workspace(cfg)
    got = dsa.topk(cfg, torch.from_numpy(sc).cuda(), ws).cpu().numpy()
    for b in range(B):
        for t in range(T):
            pos = S - T + t
            row = np.full(S, -np.inf)
            row[:pos + 1] = sc[b, t, :pos + 1]
            want, _, _ = O.dsa_select(row, topk)
            assert np.array_equal(got[b, t], want), (b, t)


@pytest.mark.parametrize("S,T", [(4000, 4), (5000, 3), (20000, 2)])
def test_topk_threshold_among_the_lowest_keys(S, T):
    """Rows whose topk-th score is -inf or the most negative finite float, so the
    radix passes' leading digits are 0 (the bin the padding past the visible keys
    also falls in): visible -inf scores before hidden keys, ties by index, on each
    register layout of the top-k."""
    rng = np.random.default_rng(S)
    sc = np.full((1, T, S), -np.inf, dtype=np.float32)
    lowest = np.float32(-3.4e38)
    for t in range(T):
        n_vis = S - T + t + 1
        n_fin = [1000, 1500, 700, 2047][t % 4]
        pick = rng.permutation(n_vis)
        sc[0, t, pick[:n_fin]] = rng.standard_normal(n_fin).astype(np.float32)
        if t % 2 == 1:  # a run of the most negative finite value straddling the threshold
            sc[0, t, pick[n_fin:n_fin + 900]] = lowest
    cfg = dsa.Config(1, T, S, topk=2048)
    ws = dsa.workspace(cfg)
    got = dsa.topk(cfg, torch.from_numpy(sc).cuda(), ws).cpu().numpy()
    for t in range(T):
        pos = S - T + t
        row = np.full(S, -np.inf)
        row[:pos + 1] = sc[0, t, :pos + 1]
        want, _, _ = O.dsa_select(row, 2048)
        assert np.array_equal(got[0, t], want), (S, t)


def test_large_cache_topk_variants():
    """Key counts for each register layout of the top-k (<= 4096, <= 16384, <= 32768)."""
    rng = np.random.default_rng(6)
    for S in (4096, 16384, 32768):
        sc = rng.standard_normal((1, 2, S)).astype(np.float32)
        cfg = dsa.Config(1, 2, S, topk=2048)
        ws = dsa.workspace(cfg)
        got = dsa.topk(cfg, torch.from_numpy(sc).cuda(), ws).cpu().numpy()
        for t in range(2):
            pos = S - 2 + t
            row = np.full(S, -np.inf)
            row[:pos + 1] = sc[0, t, :pos + 1]
            want, _, _ = O.dsa_select(row, 2048)
            assert np.array_equal(got[0, t], want), (S, t)


def test_deterministic():
    wl = W.DSA_WORKLOADS["dsa_tiny"].replace(seed=2500)
    a, b = Run(wl), Run(wl)
    assert np.array_equal(a.sel, b.sel)
    assert np.array_equal(a.scores, b.scores)


def sample_rows(wl, n, seed):
    rng = np.random.default_rng(seed)
    rows = {(0, 0), (wl.B - 1, wl.T - 1)}
    if wl.T > 2049:
        rows |= {(0, 2046), (0, 2047), (0, 2048), (wl.B - 1, 2049)}
    rows |= {(int(rng.integers(wl.B)), int(rng.integers(wl.T))) for _ in range(n)}
    return sorted(rows)


def check_sampled(wl, n, seed):
    r = Run(wl)
    assert r.device_error() == 0
    rows = sample_rows(wl, n, seed)
    n_sel = min(wl.topk, wl.S)
    for b in sorted({b for b, _ in rows}):
        ts = [t for bb, t in rows if bb == b]
        o = O.dsa_scores(r.q[b:b + 1], r.k[b:b + 1], r.w[b:b + 1]) if wl.T * wl.S <= 8192 * 512 \
            else None
        for t in ts:
            pos = wl.S - wl.T + t
            if o is None:  # one row: the oracle over this query alone, at its position
                qq, ww = r.q[b:b + 1, t:t + 1], r.w[b:b + 1, t:t + 1]
                ref = O.dsa_scores(qq, r.k[b:b + 1, :pos + 1], ww)[0, 0]
            else:
                ref = o[0, t, :pos + 1]
            bound = score_bound(r.q, r.k, r.w, [(b, t)])[0, :pos + 1]
            g = r.scores[b, t, :pos + 1].astype(np.float64)
            assert np.all(np.abs(g - ref) <= bound), (b, t)
            gs = np.full(wl.S, -np.inf)
            gs[:pos + 1] = g
            own, _, _ = O.dsa_select(gs, wl.topk)
            assert np.array_equal(r.sel[b, t], own), (b, t)
            full = np.full(wl.S, -np.inf)
            full[:pos + 1] = ref
            osel, kth, nxt = O.dsa_select(full, wl.topk)
            band = 2.0 * bound.max()
            if not np.isfinite(kth) or kth - nxt > band:
                assert np.array_equal(r.sel[b, t], osel), (b, t)
            assert len(r.sel[b, t]) == n_sel
    return r


def test_glm5_prefill_sampled():
    """4 sequences x 4096 tokens, 32 heads x 128, top 2048 (rows sampled, the
    2048-key boundary included)."""
    r = check_sampled(W.DSA_WORKLOADS["dsa_prefill"], 24, 7)
    # rows that see <= 2048 keys list keys 0 .. 2047
    assert np.array_equal(r.sel[0, 2047], np.arange(2048))
    assert not np.array_equal(r.sel[0, 2048], np.arange(2048))
    del r
    torch.cuda.empty_cache()


def test_glm5_decode_sampled():
    """64 sequences, one query each over a 32768-key cache."""
    check_sampled(W.DSA_WORKLOADS["dsa_decode"], 12, 8)
    torch.cuda.empty_cache()


def test_timeout_is_reported_and_context_survives(monkeypatch):
    """Failure detection without a GPU fault: with SRM_MOE_INJECT_STALL=1 the score
    kernel's producer arms no key copy, so the MMA warp's bounded wait on the key
    ring runs out (2 s), the kernel drains and returns, and the host reads
    MOE_ERR_TIMEOUT.  The next call on the same context is correct."""
    from sigmoid_routed_mixture_b200 import moe

    wl = W.DsaWorkload("stall", B=1, T=64, S=300, topk=32, seed=2700)
    q, k, w = W.dsa_inputs(wl)
    cfg = dsa.Config(wl.B, wl.T, wl.S, topk=wl.topk)
    ws = dsa.workspace(cfg)
    qd, kd, wd = dev_bf16(q), dev_bf16(k), torch.from_numpy(w).cuda()
    monkeypatch.setenv("SRM_MOE_INJECT_STALL", "1")
    dsa.scores(cfg, qd, kd, wd, ws)
    torch.cuda.synchronize()
    assert moe.device_error(ws) == 6  # MOE_ERR_TIMEOUT
    monkeypatch.delenv("SRM_MOE_INJECT_STALL")
    r = Run(wl)
    assert r.device_error() == 0
    r.check_rows(all_rows(wl))
