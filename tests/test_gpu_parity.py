"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on
seeded inputs, at every workload size and on the method's edge cases.
Tolerances and the near-tie rule are stated in tests/moe_harness.py."""
import gc

import numpy as np
import pytest
import torch

from oracle import oracle as O
from sigmoid_routed_mixture_b200 import moe
from sigmoid_routed_mixture_b200 import workloads as W

import moe_harness as MH

pytestmark = pytest.mark.gpu


def free():
    gc.collect()
    torch.cuda.empty_cache()


def full_check(w, forward_tokens=None):
    case = MH.Case(w)
    res = case.run()
    assert res["err"] == 0
    MH.check_route(case, res)
    MH.check_permute(case, res)
    tokens = np.arange(w.T) if forward_tokens is None else forward_tokens(res)
    rel = MH.check_forward(case, res, tokens)
    return case, res, rel


def test_tiny_full_parity():
    full_check(W.WORKLOADS["tiny"])


@pytest.mark.parametrize("T", [1, 3, 127, 129, 300])
def test_ragged_token_counts(T):
    full_check(W.WORKLOADS["tiny"].replace(T=T, seed=2000 + T))


def test_k_equals_e_dense():
    w = W.WORKLOADS["tiny"].replace(K=16, seed=2100)
    case, res, _ = full_check(w)
    assert all(sorted(r) == list(range(16)) for r in res["idx"].tolist())
    assert np.all(np.isinf(res["margin"]))


@pytest.mark.parametrize("T", [2048, 3001])
def test_cta_pair_tiles(T):
    """Enough tokens per expert (T*K >= 512*E) for the CTA-pair GEMM tiles of
    256 rows; 3001 tokens leave ragged 256-row and 128-row tails."""
    w = W.WORKLOADS["tiny"].replace(T=T, seed=2700 + T)
    assert T * w.K >= 512 * w.E
    _, res, _ = full_check(w, lambda res: MH.sample_tokens(res, w.T, 400))
    if T == 3001:  # both kinds of group end: a 128-row tail tile and a partial pair tile
        rem = np.diff(res["offsets"]) % 256
        assert np.any((rem > 0) & (rem <= 128)) and np.any(rem > 128)


@pytest.mark.parametrize("T", [300, 8192])
def test_widest_selection_256_experts_top16(T):
    """The largest supported routing: 256 experts, top-16 (the router's widest
    expert tile, 16 selection rounds, 256 groups in the permutation); 8192
    tokens give T*K = 512*E, so the CTA-pair tiles run with 257 groups."""
    w = W.WORKLOADS["tiny"].replace(E=256, K=16, T=T, seed=3300 + T)
    assert (T * w.K >= 512 * w.E) == (T == 8192)
    full_check(w, lambda res: MH.sample_tokens(res, w.T, 200))


@pytest.mark.parametrize("E,K", [(2, 1), (1, 1), (3, 2)])
def test_degenerate_expert_counts(E, K):
    """One expert per token (gate = scale), a single expert in all (every token on it)."""
    w = W.WORKLOADS["tiny"].replace(E=E, K=K, T=150, seed=3100 + 10 * E + K)
    case, res, _ = full_check(w)
    if K == 1:
        assert np.allclose(res["gate"], w.scale, rtol=0, atol=2e-6)


def test_cta_pair_tiles_without_shared_expert():
    w = W.WORKLOADS["tiny"].replace(T=2500, has_shared=False, seed=3200)
    assert w.T * w.K >= 512 * w.E
    full_check(w, lambda res: MH.sample_tokens(res, w.T, 300))


def test_without_shared_expert():
    full_check(W.WORKLOADS["tiny"].replace(has_shared=False, T=200, seed=2200))


def test_every_token_on_one_expert():
    """A large bias on expert 5 sends all 1000 tokens there: one group spans
    eight 128-row tiles with a ragged last one; other groups stay small."""
    w = W.WORKLOADS["tiny"].replace(T=1000, seed=2300)
    x, w_r, b = W.router_inputs(w)
    b[5] = 100.0
    case = MH.Case(w, x, w_r, b)
    res = case.run()
    assert res["err"] == 0
    assert res["counts"][5] == 1000
    MH.check_route(case, res)
    MH.check_permute(case, res)
    MH.check_forward(case, res, np.arange(1000))


def test_glm47flash_parity():
    w = W.WORKLOADS["glm47flash"]
    full_check(w, lambda res: MH.sample_tokens(res, w.T, 192))
    free()


def test_glm47flash_page_scale():
    """The GLM-4.7-Flash config's own routed_scaling_factor 1.8 (nnterp Config)."""
    w = W.WORKLOADS["glm47flash"].replace(T=512, scale=1.8, seed=2400)
    full_check(w, lambda res: MH.sample_tokens(res, w.T, 64))
    free()


def test_glm5_decode_parity():
    full_check(W.WORKLOADS["glm5_decode"])
    free()


@pytest.mark.parametrize("name", ["glm5_prefill", "glm5_skewed"])
def test_glm5_full_size_sampled(name):
    """Full-size launch (the benchmark's configuration); the router is compared
    on a 2048-token subset, the permutation on all tokens, the output on a
    seeded token sample that includes ragged group tails."""
    w = W.WORKLOADS[name]
    case = MH.Case(w)
    res = case.run()
    assert res["err"] == 0
    sub = np.sort(np.random.default_rng(1).choice(w.T, size=2048, replace=False))
    near = MH.check_route(case, res, sub)
    assert near < 0.05 * len(sub)
    MH.check_permute(case, res)
    MH.check_forward(case, res, MH.sample_tokens(res, w.T, 10))
    if w.skew:
        counts = res["counts"][:w.E]
        assert (counts == 0).sum() > 0      # empty groups exist
        assert counts.max() >= w.T // 2     # the top expert takes a large share
    del case, res
    free()


def test_glm5_largest_batch_sampled():
    """65536 GLM-5 tokens (four times the benchmark's batch, about 38 GB on the
    device): 512 router tiles in several waves, 524288 assignments in the
    permutation, a shared-expert group of 256 token blocks walked in chunks, and
    the index arithmetic of every stage at its largest.  Router on a 1024-token
    subset, permutation on all tokens, output on a seeded sample."""
    w = W.WORKLOADS["glm5_prefill"].replace(T=65536, seed=4500)
    case = MH.Case(w)
    res = case.run()
    assert res["err"] == 0
    sub = np.sort(np.random.default_rng(2).choice(w.T, size=1024, replace=False))
    near = MH.check_route(case, res, sub)
    assert near < 0.05 * len(sub)
    MH.check_permute(case, res)
    MH.check_forward(case, res, MH.sample_tokens(res, w.T, 6))
    del case, res
    free()


def test_ablation_uses_gates_as_given():
    """Zeroing the gates of every slot that chose expert 3 (and only those)
    changes the output exactly by those slots; zero gates leave the shared
    expert alone."""
    w = W.WORKLOADS["tiny"].replace(T=256, seed=2500)
    case = MH.Case(w)
    res = case.run()
    blk = res["block"]
    idx = res["idx"]
    assert np.any(idx == 3)
    for gate_h in (np.where(idx == 3, 0.0, res["gate"]).astype(np.float32),
                   np.zeros_like(res["gate"])):
        g_dev = torch.from_numpy(gate_h).cuda()
        y = moe.forward(case.cfg, blk.weights, case.x_dev, g_dev, blk.offsets, blk.sorted, blk.ws)
        torch.cuda.synchronize()
        y_g = MH.bf16_to_f64(y)
        y_o = case.oracle_forward(np.arange(w.T), idx, gate_h.astype(np.float64))
        assert MH.within_tolerance(y_g, y_o)[0]


def test_deterministic_and_token_permutation_invariant():
    w = W.WORKLOADS["tiny"].replace(T=300, seed=2600)
    case = MH.Case(w)
    r1 = case.run()
    r2 = case.run()
    assert np.array_equal(r1["y"], r2["y"]) and np.array_equal(r1["sorted"], r2["sorted"])
    perm = np.random.default_rng(0).permutation(w.T)
    case_p = MH.Case(w, case.x[perm], case.w_r, case.b, weights=case.weights)
    rp = case_p.run()
    assert np.array_equal(r1["idx"][perm], rp["idx"])
    assert np.array_equal(r1["gate"][perm], rp["gate"])
    assert np.array_equal(r1["y"][perm], rp["y"])


def test_zero_tokens():
    w = W.WORKLOADS["tiny"].replace(T=0)
    case = MH.Case(w)
    res = case.run()
    assert res["y"].shape == (0, w.H)
    assert np.all(res["counts"] == 0) and np.all(res["offsets"] == 0)


@pytest.mark.parametrize("T", [64, 4096, 65536])  # one-CTA, fused and three-kernel permutation
def test_out_of_range_expert_id_is_flagged(T):
    """An id past E and a negative one are flagged MOE_ERR_BAD_INDEX; the next
    call with good ids on the same workspace is exact."""
    w = W.WORKLOADS["tiny"].replace(T=T)
    cfg = moe.Config.of(w)
    g = torch.Generator(device="cuda")
    g.manual_seed(3300 + T)
    idx = torch.randint(0, w.E, (w.T, w.K), dtype=torch.int32, device="cuda", generator=g)
    bad = idx.clone()
    bad[7, 2] = w.E + 3
    bad[T - 1, 0] = -1
    ws = moe.workspace(cfg)
    moe.permute(cfg, bad, ws)
    assert moe.device_error(ws) == 5
    assert moe.device_error(ws) == 0  # read clears it
    counts, offsets, srt = moe.permute(cfg, idx, ws)
    want = O.permute(idx.cpu().numpy(), w.E, w.has_shared)
    assert moe.device_error(ws) == 0
    for got, ref in zip((counts, offsets, srt), want):
        assert np.array_equal(got.cpu().numpy(), ref)


@pytest.mark.parametrize("T,K,E,has_shared", [
    (1025, 4, 16, True),      # 5 chunks, the last one ragged: one fused launch
    (4097, 1, 7, False),      # K = 1, no shared expert
    (16384, 8, 256, True),    # the GLM-5 prefill shape: 128 chunks
    (37888, 4, 16, True),     # 148 chunks: the most one fused launch takes
    (38144, 4, 16, True),     # 149 chunks: histogram, scan and scatter kernels
])
def test_permutation_paths_match_the_oracle(T, K, E, has_shared):
    """The permutation is index work: bit-exact against the oracle's counting
    sort on either side of the fused path's chunk limit."""
    w = W.WORKLOADS["tiny"].replace(T=T, K=K, E=E, has_shared=has_shared)
    cfg = moe.Config.of(w)
    g = torch.Generator(device="cuda")
    g.manual_seed(3400 + T)
    idx = torch.randint(0, E, (T, K), dtype=torch.int32, device="cuda", generator=g)
    ws = moe.workspace(cfg)
    for _ in range(2):  # the second call reuses the workspace and its grid counter
        counts, offsets, srt = moe.permute(cfg, idx, ws)
        assert moe.device_error(ws) == 0
        want = O.permute(idx.cpu().numpy(), E, has_shared)
        for got, ref in zip((counts, offsets, srt), want):
            assert np.array_equal(got.cpu().numpy(), ref)


@pytest.mark.parametrize("T", [64, 4096])  # single-CTA tiles, CTA-pair tiles
def test_malformed_offsets_are_rejected_by_the_expert_stages(T):
    """The expert stages take offsets from the caller.  A first offset other than
    0 (the allocation-free permutation's in-band flag for a bad id), a group that
    ends before it starts, or an end past the rows gives that group no tiles and
    MOE_ERR_BAD_INDEX, with no access outside the buffers; the next call with
    good offsets is exact."""
    w = W.WORKLOADS["tiny"].replace(T=T, seed=2900 + T)
    case = MH.Case(w)
    blk = case.block()
    cfg = case.cfg
    moe.route(cfg, case.x_dev, blk.w_router, blk.bias, blk.ws, out=(blk.idx, blk.gate, blk.margin))
    moe.permute(cfg, blk.idx, blk.ws, out=(blk.counts, blk.offsets, blk.sorted))
    moe.gather_tokens(cfg, case.x_dev, blk.sorted, blk.ws)
    torch.cuda.synchronize()
    assert moe.device_error(blk.ws) == 0
    bad_idx = blk.idx.clone()
    bad_idx[3, 1] = w.E + 5
    _, flagged, _ = moe.permute_noalloc(cfg, bad_idx)
    torch.cuda.synchronize()
    assert int(flagged[0]) == -1
    good = blk.offsets.clone()
    backwards = good.clone()
    backwards[5] = backwards[4] - 1
    past_end = good.clone()
    past_end[w.E + 1] = cfg.rows + 128
    for off in (flagged, backwards, past_end):
        moe.expert_up(cfg, blk.weights, off, blk.sorted, blk.ws)
        torch.cuda.synchronize()
        assert moe.device_error(blk.ws) == 5
        moe.expert_down(cfg, blk.weights, blk.gate, off, blk.sorted, blk.ws)
        torch.cuda.synchronize()
        assert moe.device_error(blk.ws) == 5
    res = case.run()
    assert res["err"] == 0
    MH.check_forward(case, res, np.arange(w.T))


@pytest.mark.parametrize("T", [5, 300, 4096, 9600])  # split-K on single CTAs (5, 300), on CTA pairs (4096), no split (9600)
def test_route_fp32_and_packed_router_agree_bit_exact(T):
    """moe_route (fp32 W_r, split into the workspace on every call) and
    moe_pack_router + moe_route_packed run the same router kernel on the same
    split: selections, gates, margins and logits are identical."""
    w = W.WORKLOADS["glm47flash"].replace(T=T, seed=3300 + T)
    cfg = moe.Config.of(w)
    x, w_r, b = W.router_inputs(w)
    x_dev = MH.to_dev_bf16(x)
    w_r, b = torch.from_numpy(w_r).cuda(), torch.from_numpy(b).cuda()
    ws = moe.workspace(cfg)
    z1 = torch.empty((T, w.E), dtype=torch.float32, device="cuda")
    z2 = torch.empty_like(z1)
    r1 = moe.route(cfg, x_dev, w_r, b, ws, logits=z1)
    r1 = [t.clone() for t in r1]
    packed = moe.pack_router(cfg, w_r)
    r2 = moe.route_packed(cfg, x_dev, packed, b, ws, logits=z2)
    torch.cuda.synchronize()
    assert moe.device_error(ws) == 0
    for a, bb in zip(r1, r2):
        assert torch.equal(a, bb)
    assert torch.equal(z1, z2)
    case = MH.Case(w, x=x, w_r=w_r.cpu().numpy(), b=b.cpu().numpy(), weights={})
    res = dict(idx=r2[0].cpu().numpy(), gate=r2[1].cpu().numpy(), margin=r2[2].cpu().numpy(),
               logits=z2.cpu().numpy())
    tok = np.arange(T) if T <= 512 else np.random.default_rng(T).choice(T, 512, replace=False)
    MH.check_route(case, res, tok)


@pytest.mark.parametrize("T,E,K,H", [(300, 64, 3, 2048), (9600, 64, 3, 2048), (9600, 256, 9, 2048),
                                     (9600, 256, 16, 2048), (64, 256, 8, 2048), (64, 256, 16, 2048),
                                     (40, 64, 3, 2048), (64, 256, 8, 6144), (64, 256, 16, 6144)])
def test_equal_keys_take_the_lower_expert(T, E, K, H):
    """Experts 2j and 2j+1 get the same router row and bias, so their keys are
    exactly equal; the selection must take them in expert order (the lower one
    first, and never the higher one without the lower one).  Split-K router:
    one warp per token where a CTA holds several tokens (300 tokens; 64 at
    H 2048, 32 splits), the CTA-wide ranking where it holds one (64 tokens at
    H 6144, 96 splits; 40 tokens: both kinds of CTA).  9600 tokens: the
    one-pass router with its per-thread lists (K + 1 <= 9 and <= 17 entries).  The rest of the routing is checked against the oracle
    where the oracle's margin is clear."""
    w = W.WORKLOADS["glm47flash"].replace(T=T, E=E, K=K, H=H, seed=4100 + T + E + K + H)
    cfg = moe.Config.of(w)
    x, w_r, b = W.router_inputs(w)
    w_r[1::2] = w_r[0::2]
    b[1::2] = b[0::2]
    x_dev = MH.to_dev_bf16(x)
    ws = moe.workspace(cfg)
    z = torch.empty((T, E), dtype=torch.float32, device="cuda")
    packed = moe.pack_router(cfg, torch.from_numpy(w_r).cuda())
    idx, gate, margin = moe.route_packed(cfg, x_dev, packed, torch.from_numpy(b).cuda(), ws, logits=z)
    torch.cuda.synchronize()
    assert moe.device_error(ws) == 0
    z, idx, gate, margin = z.cpu().numpy(), idx.cpu().numpy(), gate.cpu().numpy(), margin.cpu().numpy()
    assert np.array_equal(z[:, 0::2].view(np.int32), z[:, 1::2].view(np.int32))
    key = (1.0 / (1.0 + np.exp(-z.astype(np.float64)))) + b.astype(np.float64)
    for t in range(T):
        sel = idx[t].tolist()
        assert len(set(sel)) == K
        for e in sel:
            if e % 2 == 1:
                assert e - 1 in sel, "token %d took expert %d without its equal %d" % (t, e, e - 1)
        for k in range(K - 1):
            a, c = sel[k], sel[k + 1]
            if a // 2 == c // 2:
                assert a < c, "token %d: equal keys out of expert order %s" % (t, sel)
            else:
                assert key[t, a] >= key[t, c] - 1e-6
    case = MH.Case(w, x=x, w_r=w_r, b=b, weights={})
    res = dict(idx=idx, gate=gate, margin=margin, logits=z)
    tok = np.arange(T) if T <= 512 else np.random.default_rng(T).choice(T, 384, replace=False)
    MH.check_route(case, res, tok)


def test_pack_reports_w2_values_fp16_cannot_hold():
    """moe_pack_weights stores W2 as fp16.  bf16 weights beyond +-65504 saturate
    and ones finer than fp16's 2^-24 spacing are rounded; the call counts them.
    The expected count is the host's own bf16 -> fp16 -> float round trip of
    every routed and shared W2 value; planted 1e5 (saturates), 1e-8 (rounds to
    0) and 3 * 2^-26 (between fp16 subnormals) must each add one, while 2^-20
    (a multiple of 2^-24) must not."""
    w = W.WORKLOADS["tiny"]
    cfg = moe.Config.of(w)
    wts = W.expert_weights(w, "cuda")

    def host_count(w2, ws2):
        a = torch.cat([w2.reshape(-1), ws2.reshape(-1)]).float().cpu()
        return int((a.half().float() != a).sum())

    n = torch.zeros((1,), dtype=torch.int32, device="cuda")
    moe.pack_weights(cfg, wts["w1"], wts["w3"], wts["w2"], wts["ws1"], wts["ws3"], wts["ws2"], inexact=n)
    torch.cuda.synchronize()
    base = host_count(wts["w2"], wts["ws2"])
    assert int(n) == base
    w2, ws2 = wts["w2"].clone(), wts["ws2"].clone()
    w2[3, 17, 5] = 1e5
    w2[0, 0, 0] = 1e-8
    ws2[9, 100] = 3 * 2.0 ** -26
    w2[5, 2, 64] = 2.0 ** -20
    expect = host_count(w2, ws2)
    planted = torch.tensor([1e5, 1e-8, 3 * 2.0 ** -26, 2.0 ** -20], dtype=torch.bfloat16).float()
    assert (planted.half().float() != planted).tolist() == [True, True, True, False]
    w13, w2p = moe.pack_weights(cfg, wts["w1"], wts["w3"], w2, wts["ws1"], wts["ws3"], ws2, inexact=n)
    torch.cuda.synchronize()
    assert int(n) == expect
    assert float(w2p[3 * w.H + 17, 5]) == 65504.0 and float(w2p[0, 0]) == 0.0
    assert float(w2p[5 * w.H + 2, 64]) == 2.0 ** -20


def test_timeout_is_reported_and_context_survives(monkeypatch):
    """Failure detection without a GPU fault: with SRM_MOE_INJECT_STALL=1 the up
    projection's producer issues no loads, so the MMA warp waits on a barrier
    nothing arms; the wait gives up after its 2 s limit, the kernel returns and
    the host reads MOE_ERR_TIMEOUT.  The next call on the same context is normal."""
    w = W.WORKLOADS["tiny"].replace(T=200, seed=2800)
    case = MH.Case(w)
    blk = case.block()
    moe.route(case.cfg, case.x_dev, blk.w_router, blk.bias, blk.ws, out=(blk.idx, blk.gate, blk.margin))
    moe.permute(case.cfg, blk.idx, blk.ws, out=(blk.counts, blk.offsets, blk.sorted))
    moe.gather_tokens(case.cfg, case.x_dev, blk.sorted, blk.ws)
    monkeypatch.setenv("SRM_MOE_INJECT_STALL", "1")
    moe.expert_up(case.cfg, blk.weights, blk.offsets, blk.sorted, blk.ws)
    torch.cuda.synchronize()
    assert moe.device_error(blk.ws) == 6  # MOE_ERR_TIMEOUT
    monkeypatch.delenv("SRM_MOE_INJECT_STALL")
    res = case.run()
    assert res["err"] == 0
    MH.check_forward(case, res, np.arange(w.T))


@pytest.mark.parametrize("name", ["tiny", "glm47flash"])
def test_rmsnorm_and_residual_sublayer(name):
    """The decoder block's FFN sublayer x' + MoE(RMSNorm(x')) ("All 43 steps"):
    the norm against the oracle's double RMSNorm (within half a bf16 ulp of the
    exact value plus fp32 rounding), the block output with the residual added
    in the combine against x' + the oracle's MoE of the same normalised rows."""
    w = W.WORKLOADS[name]
    if name == "glm47flash":
        w = w.replace(T=1024, seed=2900)
    x_res, w_r, b = W.router_inputs(w)
    gamma = W.norm_weight(w)
    case = MH.Case(w, x_res, w_r, b)
    blk = case.block()
    logits = torch.empty((w.T, w.E), dtype=torch.float32, device="cuda")
    y, x_ffn = blk.sublayer(case.x_dev, MH.to_dev_bf16(gamma), 1e-5, logits=logits)
    torch.cuda.synchronize()
    assert moe.device_error(blk.ws) == 0
    xf_bits = W.torch_bf16_to_bits(x_ffn)
    exact = O.rmsnorm(x_res, gamma, 1e-5)
    got = W.bf16_bits_to_f32(xf_bits).astype(np.float64)
    assert np.all(np.abs(got - exact) <= MH.half_ulp_bf16(exact) * 1.001 + 1e-6 * np.abs(exact))
    # the MoE on the GPU's normalised rows, selection from the GPU, gates in double
    idx = blk.idx.cpu().numpy()
    tokens = np.arange(w.T) if w.T <= 256 else np.sort(np.random.default_rng(3).choice(w.T, 128, replace=False))
    z = O.logits(xf_bits[tokens], w_r)
    gate = np.zeros(idx.shape)
    gate[tokens] = O.gates_for(z, idx[tokens], w.scale)
    norm_case = MH.Case(w, xf_bits, w_r, b, weights=case.weights)
    delta = norm_case.oracle_forward(tokens, idx, gate)
    y_o = W.bf16_bits_to_f32(x_res[tokens]).astype(np.float64) + delta
    y_g = MH.bf16_to_f64(y)[tokens]
    rms = float(np.sqrt(np.mean(delta ** 2)))
    assert np.all(np.abs(y_g - y_o) <= MH.Y_TOL * rms + MH.half_ulp_bf16(y_o))


@pytest.mark.parametrize("name,T", [("tiny_dense", 300), ("tiny_dense", 1500), ("glm47flash_dense", 4096),
                                    ("glm5_dense", 16384)])
def test_dense_mlp(name, T):
    """The dense SwiGLU MLP of the first blocks through the same kernels as one
    group (E = K = 0): against the oracle's shared-expert SwiGLU (a single dummy
    routed expert at gate 0 leaves exactly the shared term), with the residual
    added in the combine."""
    if name == "tiny_dense":
        w = W.WORKLOADS["tiny"].replace(name="tiny_dense", T=T, I=512, E=0, K=0, seed=3000 + T)
    else:
        w = W.WORKLOADS[name]
    rng = np.random.default_rng(w.seed)
    x = W.f32_to_bf16_bits(rng.standard_normal((w.T, w.H), dtype=np.float32))
    res = W.f32_to_bf16_bits(rng.standard_normal((w.T, w.H), dtype=np.float32))
    wt = W.expert_weights(w, "cuda")
    cfg = moe.Config.dense(w.T, w.H, w.I)
    weights = moe.pack_weights(cfg, None, None, None, wt["ws1"], wt["ws3"], wt["ws2"])
    ws = moe.workspace(cfg)
    y = moe.dense_mlp(cfg, weights, MH.to_dev_bf16(x), ws, residual=MH.to_dev_bf16(res))
    torch.cuda.synchronize()
    assert moe.device_error(ws) == 0
    tokens = np.arange(w.T) if w.T <= 1500 else np.sort(rng.choice(w.T, 24, replace=False))
    sh = [W.torch_bf16_to_bits(wt[n]) for n in ("ws1", "ws3", "ws2")]
    dummy1 = [np.zeros((w.I, w.H), np.uint16)]
    dummy2 = [np.zeros((w.H, w.I), np.uint16)]
    idx = np.zeros((w.T, 1), np.int32)
    mlp = O.forward(x, dummy1, dummy1, dummy2, sh[0], sh[1], sh[2], idx, np.zeros((w.T, 1)), tokens=tokens)
    y_o = W.bf16_bits_to_f32(res[tokens]).astype(np.float64) + mlp
    y_g = MH.bf16_to_f64(y)[tokens]
    rms = float(np.sqrt(np.mean(mlp ** 2)))
    assert np.all(np.abs(y_g - y_o) <= MH.Y_TOL * rms + MH.half_ulp_bf16(y_o))
    del wt, weights, ws
    free()
