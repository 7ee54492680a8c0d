"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
on a seeded workload and compare it with the CPU oracle.

Acceptance rules (the layer's own tolerance, written here once):
  * selection: identical expert sets on every token whose oracle margin
    (K-th minus (K+1)-th key of s + b) exceeds MARGIN_TOL; tokens at or under
    it are near ties, where either choice is correct: they are excluded from
    the index comparison and counted;
  * permutation: counts / offsets / sorted bit-identical to the oracle's
    counting sort of the GPU's own indices;
  * logits: |z_gpu - z_oracle| <= Z_TOL * (1 + max|z|) (fp32-accurate);
  * slot order: descending exact key, except between selected keys closer
    than ORDER_TOL (within the router's precision either order is correct);
  * gates: |G_gpu - G_oracle| <= GATE_TOL per expert on tokens with equal sets;
  * output: |y_gpu - y_oracle| <= Y_TOL * RMS(y_oracle) + half_ulp_bf16(y_oracle)
    element by element, where the oracle is exact (double) and uses the GPU's
    selection with gates recomputed in double.  The half-ulp term is the
    representation error of the bf16 result itself, which no implementation
    avoids: for |y| in [16, 32) it is 0.0625, more than 2e-2 x RMS whenever
    RMS < 3.1.  The raw max |y_gpu - y_oracle| / RMS is returned for reporting.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import oracle as O
from sigmoid_routed_mixture_b200 import moe
from sigmoid_routed_mixture_b200 import workloads as W

MARGIN_TOL = 1e-4
Z_TOL = 2e-6
ORDER_TOL = 1e-5
GATE_TOL = 2e-5
Y_TOL = 2e-2


def to_dev_bf16(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def half_ulp_bf16(v: np.ndarray) -> np.ndarray:
    """Half the spacing of bf16 numbers at |v| (8 significant bits)."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, np.finfo(np.float64).tiny)))
    return np.where(a > 0, np.exp2(e - 8), 0.0)


def within_tolerance(y_g, y_o):
    """(ok, raw max|dy|/rms, worst excess) under the output rule above."""
    rms = float(np.sqrt(np.mean(y_o ** 2)))
    err = np.abs(y_g - y_o)
    bound = Y_TOL * rms + half_ulp_bf16(y_o)
    return bool(np.all(err <= bound)), float(err.max() / rms) if rms > 0 else 0.0, float((err - bound).max())


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return W.bf16_bits_to_f32(W.torch_bf16_to_bits(t)).astype(np.float64)


class Case:
    """Inputs of one workload on the GPU (router inputs also kept on the host)."""

    def __init__(self, w: W.Workload, x=None, w_r=None, b=None, weights=None):
        self.w = w
        if x is None:
            x, w_r, b = W.router_inputs(w)
        self.x, self.w_r, self.b = x, w_r, b
        self.weights = weights if weights is not None else W.expert_weights(w, "cuda")
        self.cfg = moe.Config.of(w)
        self.x_dev = to_dev_bf16(x)
        self.w_r_dev = torch.from_numpy(w_r).cuda()
        self.b_dev = torch.from_numpy(b).cuda()
        self._host_w = {}

    def block(self):
        wt = self.weights
        return moe.MoeBlock(self.cfg, self.w_r_dev, self.b_dev, wt["w1"], wt["w3"], wt["w2"],
                            wt.get("ws1"), wt.get("ws3"), wt.get("ws2"))

    def run(self):
        """Route + permute + forward on the GPU; returns host copies of every output."""
        blk = self.block()
        logits = torch.empty((self.w.T, self.w.E), dtype=torch.float32, device="cuda")
        y = blk(self.x_dev, logits=logits)
        torch.cuda.synchronize()
        err = moe.device_error(blk.ws)
        return dict(idx=blk.idx.cpu().numpy(), gate=blk.gate.cpu().numpy(),
                    margin=blk.margin.cpu().numpy(), counts=blk.counts.cpu().numpy(),
                    offsets=blk.offsets.cpu().numpy(), sorted=blk.sorted.cpu().numpy(),
                    y=bf16_to_f64(y), logits=logits.cpu().numpy(), err=err, block=blk)

    def host_expert(self, name, e):
        key = (name, e)
        if key not in self._host_w:
            self._host_w[key] = W.torch_bf16_to_bits(self.weights[name][e])
        return self._host_w[key]

    def oracle_tables(self, experts):
        E = self.w.E
        t1 = [self.host_expert("w1", e) if e in experts else None for e in range(E)]
        t3 = [self.host_expert("w3", e) if e in experts else None for e in range(E)]
        t2 = [self.host_expert("w2", e) if e in experts else None for e in range(E)]
        if self.w.has_shared:
            sh = [W.torch_bf16_to_bits(self.weights[n]) for n in ("ws1", "ws3", "ws2")]
        else:
            sh = [None, None, None]
        return t1, t3, t2, sh

    def oracle_forward(self, tokens, idx, gate):
        """Oracle y for the listed tokens with the given selection and gates."""
        tokens = np.asarray(tokens, dtype=np.int64)
        experts = set(np.unique(idx[tokens]).tolist())
        t1, t3, t2, sh = self.oracle_tables(experts)
        return O.forward(self.x, t1, t3, t2, sh[0], sh[1], sh[2], idx, gate, tokens=tokens,
                         has_shared=self.w.has_shared)


def check_route(case: Case, res, tokens=None):
    """Selection, gate and margin parity on `tokens` (all when None); returns near-tie count."""
    w = case.w
    tok = np.arange(w.T) if tokens is None else np.asarray(tokens)
    idx_o, gate_o, margin_o, z_o = O.route(case.x[tok], case.w_r, case.b, w.K, w.scale)
    # logits: fp32-accurate (three-part split of W_r, fp32 accumulation)
    dz = np.abs(res["logits"][tok] - z_o)
    assert dz.max() <= Z_TOL * (1.0 + np.abs(z_o).max()), "router logits off by %g" % dz.max()
    idx_g, gate_g, margin_g = res["idx"][tok], res["gate"][tok], res["margin"][tok]
    clear = margin_o > MARGIN_TOL
    near = int((~clear).sum())
    for r in np.nonzero(clear)[0]:
        assert sorted(idx_g[r].tolist()) == sorted(idx_o[r].tolist()), (
            "token %d: gpu %s oracle %s margin %g" % (tok[r], idx_g[r], idx_o[r], margin_o[r]))
        go = dict(zip(idx_o[r].tolist(), gate_o[r].tolist()))
        for k in range(w.K):
            assert abs(gate_g[r, k] - go[int(idx_g[r, k])]) <= GATE_TOL
    # slot order: descending key where the oracle's adjacent keys are clearly apart
    key_o = 1.0 / (1.0 + np.exp(-z_o)) + case.b.astype(np.float64)
    for r in np.nonzero(clear)[0]:
        ks = key_o[r, idx_g[r]]
        assert np.all(np.diff(ks) <= ORDER_TOL), "slot order not descending at token %d" % tok[r]
    # gates sum to the scale; margins agree where the GPU saw the same choice
    assert np.max(np.abs(gate_g.sum(axis=1) - w.scale)) <= 8 * w.K * np.spacing(np.float32(w.scale))
    finite = np.isfinite(margin_o) & clear
    if finite.any():
        assert np.max(np.abs(margin_g[finite] - margin_o[finite])) <= 1e-5
    assert np.all(np.isinf(margin_g[~np.isfinite(margin_o)]))
    return near


def check_permute(case: Case, res):
    counts, offsets, srt = O.permute(res["idx"], case.w.E, case.w.has_shared)
    assert np.array_equal(res["counts"], counts)
    assert np.array_equal(res["offsets"], offsets)
    assert np.array_equal(res["sorted"], srt)


def check_forward(case: Case, res, tokens):
    """End-to-end output parity on `tokens`: oracle with the GPU's selection and
    double-precision gates of that selection."""
    tokens = np.asarray(tokens, dtype=np.int64)
    z = O.logits(case.x, case.w_r) if case.w.T <= 4096 else None
    idx = res["idx"]
    if z is None:
        gate = np.zeros(idx.shape, dtype=np.float64)
        zt = O.logits(case.x[tokens], case.w_r)
        gate[tokens] = O.gates_for(zt, idx[tokens], case.w.scale)
    else:
        gate = O.gates_for(z, idx, case.w.scale)
    y_o = case.oracle_forward(tokens, idx, gate)
    y_g = res["y"][tokens]
    assert np.sqrt(np.mean(y_o ** 2)) > 0
    ok, rel, excess = within_tolerance(y_g, y_o)
    assert ok, "output outside 2e-2*rms + half-ulp: max|dy|/rms %g, worst excess %g" % (rel, excess)
    return rel


def sample_tokens(res, T, n_random, seed=0):
    """A seeded token sample that always includes the first and last token, the
    tokens in the ragged last row of the largest expert groups, and the tokens
    on either side of each group's last 256-row boundary."""
    rng = np.random.default_rng(seed)
    picks = {0, T - 1}
    picks.update(rng.choice(T, size=min(n_random, T), replace=False).tolist())
    offsets, srt = res["offsets"], res["sorted"]
    K = res["idx"].shape[1]
    counts = np.diff(offsets)[:-1]
    rows = []
    for g in np.argsort(-counts)[:4]:
        if counts[g] > 0:
            rows.append(offsets[g + 1] - 1)
    # Both ways a group can end in 256-row CTA-pair tiling: a last partial
    # block of <= 128 rows (its own 128-row tile) or of 129..255 rows (a
    # partial pair tile).  Take the rows on either side of each boundary, for
    # up to 16 groups of each kind.
    n_groups = len(offsets) - 1  # routed experts and the shared expert
    kinds = {True: 0, False: 0}
    for g in range(n_groups):
        c = int(offsets[g + 1] - offsets[g])
        if c % 256 == 0:
            continue
        small = c % 256 <= 128
        if kinds[small] >= 16:
            continue
        kinds[small] += 1
        start = int(offsets[g]) + c // 256 * 256
        rows += [start, int(offsets[g + 1]) - 1] + ([start - 1] if c >= 256 else [])
    for r in rows:
        a = int(srt[r])
        picks.add(a // K if a < T * K else a - T * K)
    return np.array(sorted(picks), dtype=np.int64)
