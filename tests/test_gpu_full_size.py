"""Parity at the benchmark workloads' own sizes, in the launch configuration
the benchmark times, on outputs the fp64 oracle can compute one by one.

* scan_128k: the selective scan alone, batch 1, L = 131072, d_inner 8192,
  automatic time chunks; sampled channels element by element (one bf16 step)
  and their final state.
* decode_b64: 2048-token prefill of 64 rows, then 1024 one-token steps
  replayed from one CUDA graph; every step of three sampled rows against the
  oracle's prefill of the same 3072 tokens (decode step == prefill of L + 1).
* layer_pair: 4 x 8192 tokens, Mamba + 16-expert top-2 MoE with bf16
  experts at d_ff 14336; every router decision bit-exact on the GPU's own
  router input, the end-to-end decisions of one batch row against the fp64
  pair away from near-ties, and 48 sampled tokens' outputs.
Batch rows and channels are independent, so sampling them is exact.
"""
import numpy as np
import pytest
import torch

from oracle import mamba as om
from oracle import moe as omoe
from synthetic import MoEShape, block_norm_params, decode_inputs, mamba_input, mamba_params, moe_params, \
    scan_inputs, workload
from tests.helpers import TOL_BF16, cuda_or_skip, rel_l2, to_np

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def dev():
    d = cuda_or_skip()
    import mamba_selective_scan_mixer_b200 as J
    J.lib()
    return d


class _ExpertsFp64:
    """Expert weights widened to fp64 one expert at a time, when the oracle asks for them."""

    def __init__(self, t):
        self.t = t

    def __getitem__(self, e):
        return to_np(self.t[e])


def _near_ties(logits, k, rel):
    s = -np.sort(-logits, axis=1)
    scale = np.abs(logits).max(axis=1)
    gaps = np.diff(s[:, :k + 1], axis=1)
    return np.nonzero((np.abs(gaps) < rel * scale[:, None]).any(axis=1))[0]


def test_scan_128k_full_size_sampled_channels(dev):
    import mamba_selective_scan_mixer_b200 as J
    wl = workload("scan_128k")
    L, di = wl["seqlen"], wl["d_inner"]
    s = scan_inputs(1, L, di, 16, seed=0, device=dev)      # the benchmark's own draws
    y, h = J.selective_scan(s["x"], s["z"], s["dt"], s["B"], s["C"], s["A"], s["D"])
    J.device_status()
    rng = np.random.default_rng(3)
    cols = np.sort(rng.choice(di, 200, replace=False))
    ci = torch.as_tensor(cols, device=dev)
    n = lambda t: to_np(t.index_select(-1, ci)) if t.shape[-1] == di else to_np(t)
    wy, wh = om.selective_scan_c(n(s["x"]), n(s["dt"]), to_np(s["A"][ci]), n(s["B"]), n(s["C"]),
                                 to_np(s["D"][ci]), n(s["z"]))
    got = n(y)
    scale = np.sqrt(np.mean(wy ** 2))
    bad = np.abs(got - wy) > 2.0 ** -7 * np.abs(wy) + 1e-5 * scale
    assert int(bad.sum()) == 0, np.argwhere(bad)[:5]
    assert rel_l2(got, wy) < TOL_BF16
    assert rel_l2(to_np(h[:, ci]), wh) < 1e-5


def test_decode_b64_graph_1024_steps(dev):
    import mamba_selective_scan_mixer_b200 as J
    wl = workload("decode_b64")
    sh = wl["mamba"]
    B, L0, S = wl["batch"], wl["prefill"], wl["steps"]
    params = mamba_params(sh, seed=0)
    mixer = J.MambaMixer({k: v.to(dev) for k, v in params.items()}, sh)
    u0 = mamba_input(sh, B, L0, seed=1, device=dev)
    cs, ss = mixer.new_states(B)
    mixer.prefill(u0, conv_state_out=cs, ssm_state_out=ss)
    steps_u = decode_inputs(sh, B, S, seed=1, device=dev)
    outs = torch.empty(S, B, sh.d_model, dtype=torch.bfloat16, device=dev)
    scs, sss = cs.clone(), ss.clone()
    mixer.step(steps_u[0], scs, sss, out=outs[0])           # sizes the workspace before capture
    torch.cuda.synchronize()
    gs = torch.cuda.Stream(dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=gs):
        for t in range(S):
            mixer.step(steps_u[t], cs, ss, out=outs[t])
    graph.replay()
    torch.cuda.synchronize()
    J.device_status()
    rows = [0, 37, 63]
    ri = torch.as_tensor(rows, device=dev)
    full = torch.cat([u0.index_select(0, ri), steps_u.index_select(1, ri).transpose(0, 1)], dim=1)
    ref = om.mamba_prefill(om.params64(params), to_np(full), sh, scan="c")
    got = to_np(outs.index_select(1, ri).transpose(0, 1))
    assert rel_l2(got, ref["out"][:, L0:]) < TOL_BF16
    # per step too, so that no stretch of the 1024 steps can hide in the norm
    per_step = [rel_l2(got[:, t], ref["out"][:, L0 + t]) for t in range(S)]
    assert max(per_step) < 2 * TOL_BF16, int(np.argmax(per_step))
    assert rel_l2(to_np(ss.index_select(0, ri)), ref["ssm_state"]) < TOL_BF16
    assert rel_l2(to_np(cs.index_select(0, ri)), ref["conv_state"]) < TOL_BF16
    del graph


def test_layer_pair_full_size_bf16_experts(dev):
    import mamba_selective_scan_mixer_b200 as J
    wl = workload("layer_pair")
    sh, es = wl["mamba"], wl["moe"]
    B, L = wl["batch"], wl["seqlen"]
    mp = mamba_params(sh, seed=0)
    ep = moe_params(es, seed=0, device=dev)
    mixer = J.MambaMixer({k: v.to(dev) for k, v in mp.items()}, sh)
    moe = J.MoE(ep, es)
    g1, g2 = block_norm_params(sh.d_model, device=dev)
    x = mamba_input(sh, B, L, seed=2, device=dev)
    r = J.layer_pair(mixer, moe, x, g1, g2)
    torch.cuda.synchronize()
    J.device_status()
    # every router decision bit-exact on the router input the GPU fed its MoE
    v = J.rmsnorm(r["h"].view(B * L, sh.d_model), g2, 1e-6)
    idx, w, logits = omoe.router(to_np(v), to_np(ep["router"]), es.top_k)
    assert len(_near_ties(logits, es.top_k, 1e-12)) == 0
    np.testing.assert_array_equal(r["idx"].cpu().numpy(), idx)
    counts = np.bincount(idx.reshape(-1), minlength=es.n_experts)
    np.testing.assert_array_equal(np.diff(r["offsets"].cpu().numpy()), counts)
    # end to end on batch row 1 against the fp64 pair
    b = 1
    rng = np.random.default_rng(5)
    tok = np.sort(rng.choice(L, 48, replace=False))
    ep64 = {"router": to_np(ep["router"]), **{k: _ExpertsFp64(ep[k]) for k in ("w_gate", "w_up", "w_down")}}
    want = omoe.layer_pair(om.params64(mp), ep64, to_np(x[b:b + 1]), sh, es.top_k, to_np(g1), to_np(g2),
                           tokens=tok, scan="c")
    got_h = to_np(r["h"][b])
    assert rel_l2(got_h, want["h"]) < TOL_BF16
    # the oracle's router on its own fp64 input: decisions agree away from near-ties
    ok = np.setdiff1d(np.arange(L), _near_ties(want["logits"], es.top_k, 2e-2))
    assert len(ok) > L // 2
    np.testing.assert_array_equal(r["idx"].cpu().numpy()[b * L + ok], want["idx"][ok])
    got = to_np(r["out"][torch.as_tensor(b * L + tok, device=dev)])
    assert rel_l2(got, want["out"]) < TOL_BF16
