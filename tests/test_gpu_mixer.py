"""Mamba mixer parity through the C ABI: prefill, decode step, caches and the
step-equals-prefill property, against the fp64 oracle on seeded inputs."""
import numpy as np
import pytest
import torch

from oracle import mamba as om
from synthetic import MambaShape, decode_inputs, mamba_input, mamba_params, workload
from tests.helpers import TOL_BF16, TOL_F32, bf16_steps, cuda_or_skip, rel_l2, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    d = cuda_or_skip()
    import mamba_selective_scan_mixer_b200 as J
    J.lib()
    return d


def _mixer(shape, seed, dev, **kw):
    import mamba_selective_scan_mixer_b200 as J
    p = mamba_params(shape, seed=seed, **kw)
    return J.MambaMixer({k: v.to(dev) for k, v in p.items()}, shape), om.params64(p)


def test_tiny_fp32_prefill_and_16_steps(dev):
    """tiny fp32 mixer: prefill of 256 tokens then 16 decode steps, fp32 bar"""
    wl = workload("tiny_fp32")
    sh = wl["mamba"]
    mix, p64 = _mixer(sh, 0, dev)
    u = mamba_input(sh, 1, wl["seqlen"] + wl["steps"], seed=0)
    u64 = to_np(u)
    out, cs, ss = mix.prefill(u[:, :wl["seqlen"]].contiguous().to(dev))
    ref = om.mamba_prefill(p64, u64[:, :wl["seqlen"]], sh)
    assert rel_l2(to_np(out), ref["out"]) < TOL_F32
    assert rel_l2(to_np(cs), ref["conv_state"]) < TOL_F32
    assert rel_l2(to_np(ss), ref["ssm_state"]) < TOL_F32
    rcs, rss = ref["conv_state"], ref["ssm_state"]
    outs, wants = [], []
    for t in range(wl["steps"]):
        o = mix.step(u[:, wl["seqlen"] + t].contiguous().to(dev), cs, ss)
        w, rcs, rss = om.mamba_step(p64, u64[:, wl["seqlen"] + t], sh, rcs, rss)
        outs.append(to_np(o))
        wants.append(w)
    assert rel_l2(np.stack(outs), np.stack(wants)) < TOL_F32
    assert rel_l2(to_np(ss), rss) < TOL_F32
    assert rel_l2(to_np(cs), rcs) < TOL_F32


@pytest.mark.parametrize("inner_norm", [True, False])
def test_bf16_prefill_small_widths(dev, inner_norm):
    sh = MambaShape(d_model=256, d_inner=512, dt_rank=32, dtype="bf16", inner_norm=inner_norm)
    mix, p64 = _mixer(sh, 1, dev, norm_init="random", d_init="random")
    u = mamba_input(sh, 2, 300, seed=1)
    out, cs, ss = mix.prefill(u.to(dev))
    ref = om.mamba_prefill(p64, to_np(u), sh)
    assert rel_l2(to_np(out), ref["out"]) < TOL_BF16
    assert rel_l2(to_np(ss), ref["ssm_state"]) < TOL_BF16
    assert rel_l2(to_np(cs), ref["conv_state"]) < TOL_BF16


def test_bf16_prefill_residual_and_continuation(dev):
    """prefill continues from given caches; residual added in the out_proj epilogue"""
    sh = MambaShape(d_model=256, d_inner=512, dt_rank=32, dtype="bf16")
    mix, p64 = _mixer(sh, 2, dev, a_init="random")
    u = mamba_input(sh, 1, 200, seed=2)
    res = mamba_input(sh, 1, 200, seed=3)
    ud = u.to(dev)
    _, cs, ss = mix.prefill(ud[:, :120].contiguous())
    out, cs2, ss2 = mix.prefill(ud[:, 120:].contiguous(), residual=res[:, 120:].contiguous().to(dev),
                                conv_state_in=cs, ssm_state_in=ss)
    ref = om.mamba_prefill(p64, to_np(u), sh)
    assert rel_l2(to_np(out), ref["out"][:, 120:] + to_np(res)[:, 120:]) < TOL_BF16
    assert rel_l2(to_np(ss2), ref["ssm_state"]) < TOL_BF16
    # in-place continuation: caches in == out
    cs3, ss3 = cs.clone(), ss.clone()
    mix.prefill(ud[:, 120:].contiguous(), conv_state_in=cs3, ssm_state_in=ss3, conv_state_out=cs3,
                ssm_state_out=ss3)
    assert torch.equal(cs3, cs2)
    assert rel_l2(to_np(ss3), to_np(ss2)) < 1e-6


def test_bf16_prefill_reordered_channel_groups(dev):
    """d_inner 2048: eight scan groups of 256 channels after the bf16 handle
    reorders its channels by decay speed, each group with its own number of
    time chunks; 1200 tokens in two calls (the second from the first's
    caches), outputs and both caches in the caller's channel order"""
    sh = MambaShape(d_model=512, d_inner=2048, dt_rank=64, dtype="bf16", inner_norm=True)
    mix, p64 = _mixer(sh, 12, dev, a_init="structured", norm_init="random")
    u = mamba_input(sh, 2, 1200, seed=12)
    ud = u.to(dev)
    out1, cs, ss = mix.prefill(ud[:, :700].contiguous())
    out2, cs2, ss2 = mix.prefill(ud[:, 700:].contiguous(), conv_state_in=cs, ssm_state_in=ss)
    ref = om.mamba_prefill(p64, to_np(u), sh)
    assert rel_l2(np.concatenate([to_np(out1), to_np(out2)], axis=1), ref["out"]) < TOL_BF16
    assert rel_l2(to_np(ss2), ref["ssm_state"]) < TOL_BF16
    assert rel_l2(to_np(cs2), ref["conv_state"]) < TOL_BF16
    # in-place continuation over many time chunks: the state in is copied
    # before the scan (its first chunk reads it while its last chunk writes
    # it), so the result is the continuation into separate caches (up to the
    # rounding order of the carries, which the look-back takes as they come)
    cs3, ss3 = cs.clone(), ss.clone()
    out3, _, _ = mix.prefill(ud[:, 700:].contiguous(), conv_state_in=cs3, ssm_state_in=ss3, conv_state_out=cs3,
                             ssm_state_out=ss3)
    assert bf16_steps(to_np(out3), to_np(out2)) <= 1
    assert rel_l2(to_np(ss3), to_np(ss2)) < 1e-6
    assert torch.equal(cs3, cs2)


def test_bf16_decode_steps_match_oracle_and_prefill(dev):
    sh = MambaShape(d_model=512, d_inner=1024, dt_rank=64, dtype="bf16")
    mix, p64 = _mixer(sh, 4, dev)
    B, L0, S = 5, 40, 12
    u = mamba_input(sh, B, L0, seed=4)
    steps = decode_inputs(sh, B, S, seed=4)
    _, cs, ss = mix.prefill(u.to(dev))
    outs = [to_np(mix.step(steps[t].to(dev), cs, ss)) for t in range(S)]
    full = torch.cat([u, steps.transpose(0, 1)], dim=1)
    ref = om.mamba_prefill(p64, to_np(full), sh)
    assert rel_l2(np.stack(outs, 1), ref["out"][:, L0:]) < TOL_BF16
    assert rel_l2(to_np(ss), ref["ssm_state"]) < TOL_BF16
    # GPU step == GPU prefill of the longer sequence
    out_full, _, ss_full = mix.prefill(full.contiguous().to(dev))
    assert rel_l2(np.stack(outs, 1), to_np(out_full)[:, L0:]) < TOL_BF16


@pytest.mark.parametrize("dt_rank,batch,inner_norm,a_init", [
    (64, 5, True, "structured"),
    (64, 64, False, "random"),      # no inner norm, per-state decays
    (64, 1, True, "random"),        # one row
    (40, 5, True, "structured"),    # dt_rank not a multiple of 32
    (64, 65, True, "structured"),   # odd batch above 64
])
def test_bf16_decode_shapes(dev, dt_rank, batch, inner_norm, a_init):
    """decode steps against the oracle across batch sizes, dt ranks, norm and
    A variants, caches included"""
    sh = MambaShape(d_model=256, d_inner=1024, dt_rank=dt_rank, dtype="bf16", inner_norm=inner_norm)
    mix, p64 = _mixer(sh, 6, dev, a_init=a_init, norm_init="random")
    L0, S = 24, 6
    u = mamba_input(sh, batch, L0, seed=6)
    steps = decode_inputs(sh, batch, S, seed=6)
    _, cs, ss = mix.prefill(u.to(dev))
    outs = [to_np(mix.step(steps[t].to(dev), cs, ss)) for t in range(S)]
    full = torch.cat([u, steps.transpose(0, 1)], dim=1)
    ref = om.mamba_prefill(p64, to_np(full), sh)
    assert rel_l2(np.stack(outs, 1), ref["out"][:, L0:]) < TOL_BF16
    assert rel_l2(to_np(ss), ref["ssm_state"]) < TOL_BF16
    assert rel_l2(to_np(cs), ref["conv_state"]) < TOL_BF16


@pytest.mark.parametrize("batch", [65, 7])
def test_bf16_decode_residual(dev, batch):
    """decode steps with a residual (added in the split-K sum of out_proj;
    batch 65: a ragged second token tile) and without one, against the
    oracle; the caches are the same either way"""
    sh = MambaShape(d_model=512, d_inner=1024, dt_rank=64, dtype="bf16", inner_norm=True)
    mix, p64 = _mixer(sh, 17, dev, a_init="random", norm_init="random")
    L0, S = 16, 4
    u = mamba_input(sh, batch, L0, seed=17)
    steps = decode_inputs(sh, batch, S, seed=17)
    res = decode_inputs(sh, batch, S, seed=18)
    _, cs, ss = mix.prefill(u.to(dev))
    cs2, ss2 = cs.clone(), ss.clone()
    outs, plain = [], []
    for t in range(S):
        outs.append(to_np(mix.step(steps[t].to(dev), cs, ss, residual=res[t].to(dev))))
        plain.append(to_np(mix.step(steps[t].to(dev), cs2, ss2)))
    full = torch.cat([u, steps.transpose(0, 1)], dim=1)
    ref = om.mamba_prefill(p64, to_np(full), sh)
    want = ref["out"][:, L0:] + np.stack([to_np(r) for r in res], 1)
    assert rel_l2(np.stack(outs, 1), want) < TOL_BF16
    assert rel_l2(np.stack(plain, 1), ref["out"][:, L0:]) < TOL_BF16
    assert torch.equal(ss, ss2) and torch.equal(cs, cs2)


def test_bf16_decode_mid_width(dev):
    """d_model 1024 / d_inner 2048, batch 8: the decode GEMMs at a width
    between the small cases and Jamba's"""
    sh = MambaShape(d_model=1024, d_inner=2048, dt_rank=64, dtype="bf16", inner_norm=True)
    mix, p64 = _mixer(sh, 10, dev, a_init="structured", norm_init="random")
    L0, S, batch = 16, 4, 8
    u = mamba_input(sh, batch, L0, seed=10)
    steps = decode_inputs(sh, batch, S, seed=10)
    _, cs, ss = mix.prefill(u.to(dev))
    outs = [to_np(mix.step(steps[t].to(dev), cs, ss)) for t in range(S)]
    full = torch.cat([u, steps.transpose(0, 1)], dim=1)
    ref = om.mamba_prefill(p64, to_np(full), sh)
    assert rel_l2(np.stack(outs, 1), ref["out"][:, L0:]) < TOL_BF16
    assert rel_l2(to_np(ss), ref["ssm_state"]) < TOL_BF16


def test_bf16_decode_ragged_width(dev):
    """d_inner 136 (not a multiple of 64) at batch 3: 408 (row, channel) pairs,
    so the last block of the state update is partly empty"""
    sh = MambaShape(d_model=128, d_inner=136, dt_rank=8, dtype="bf16", inner_norm=True)
    mix, p64 = _mixer(sh, 9, dev, a_init="random", norm_init="random")
    L0, S, batch = 20, 5, 3
    u = mamba_input(sh, batch, L0, seed=9)
    steps = decode_inputs(sh, batch, S, seed=9)
    _, cs, ss = mix.prefill(u.to(dev))
    outs = [to_np(mix.step(steps[t].to(dev), cs, ss)) for t in range(S)]
    full = torch.cat([u, steps.transpose(0, 1)], dim=1)
    ref = om.mamba_prefill(p64, to_np(full), sh)
    assert rel_l2(np.stack(outs, 1), ref["out"][:, L0:]) < TOL_BF16
    assert rel_l2(to_np(ss), ref["ssm_state"]) < TOL_BF16
    assert rel_l2(to_np(cs), ref["conv_state"]) < TOL_BF16


@pytest.mark.parametrize("L,chunk", [(200, 48), (300, 64)])
def test_prefill_from_host_memory_pipelined(dev, L, chunk):
    """the host-buffer prefill (transfers overlapped with compute in time
    chunks: uniform with a ragged tail, or ramped at both ends; residual
    aliasing the output) equals the device prefill and the oracle"""
    sh = MambaShape(d_model=256, d_inner=512, dt_rank=32, dtype="bf16")
    mix, p64 = _mixer(sh, 7, dev, a_init="random")
    B = 2
    u = mamba_input(sh, B, L, seed=8)
    res = mamba_input(sh, B, L, seed=9)
    cs0, ss0 = mix.new_states(B)
    cs0.normal_()
    ss0.normal_()
    cs0 = cs0.to(torch.bfloat16).float()   # the cache holds bf16 values
    want, wcs, wss = mix.prefill(u.to(dev), residual=res.to(dev), conv_state_in=cs0, ssm_state_in=ss0)
    hu = u.clone().pin_memory()
    hres = res.clone().pin_memory()
    out, cs, ss = mix.prefill_host(hu, residual_host=hres, out_host=hres, chunk=chunk, conv_state_in=cs0,
                                   ssm_state_in=ss0)
    torch.cuda.synchronize()
    assert out.data_ptr() == hres.data_ptr()
    assert rel_l2(to_np(out), to_np(want)) < TOL_BF16
    assert rel_l2(to_np(cs), to_np(wcs)) < 1e-6
    assert rel_l2(to_np(ss), to_np(wss)) < 1e-4
    ref = om.mamba_prefill(p64, to_np(u), sh, conv_state0=to_np(cs0), ssm_state0=to_np(ss0))
    assert rel_l2(to_np(out), ref["out"] + to_np(res)) < TOL_BF16
    # pageable host memory is refused
    with pytest.raises(ValueError):
        mix.prefill_host(u.clone())


@pytest.mark.slow
def test_prefill_4k_full_width(dev):
    """Jamba-width prefill of 4096 tokens with inner RMSNorm, whole output vs the oracle"""
    wl = workload("prefill_4k")
    sh = wl["mamba"]
    mix, p64 = _mixer(sh, 0, dev)
    u = mamba_input(sh, wl["batch"], wl["seqlen"], seed=0)
    out, cs, ss = mix.prefill(u.to(dev))
    ref = om.mamba_prefill(p64, to_np(u), sh, scan="c")
    assert rel_l2(to_np(out), ref["out"]) < TOL_BF16
    assert rel_l2(to_np(ss), ref["ssm_state"]) < TOL_BF16


@pytest.mark.slow
def test_decode_b64_full_width_sampled_rows(dev):
    """batch-64 decode at Jamba width: 2048-token prefill then steps; sampled batch
    rows checked against the oracle's prefill of the same token sequence"""
    wl = workload("decode_b64")
    sh = wl["mamba"]
    mix, p64 = _mixer(sh, 0, dev)
    B, L0, S = wl["batch"], wl["prefill"], 32
    u = mamba_input(sh, B, L0, seed=0)
    steps = decode_inputs(sh, B, S, seed=0)
    _, cs, ss = mix.prefill(u.to(dev))
    sd = steps.to(dev)
    outs = torch.stack([mix.step(sd[t], cs, ss) for t in range(S)], 1)
    rows = [0, 37, 63]
    full = torch.cat([u[rows], steps[:, rows].transpose(0, 1)], dim=1)
    ref = om.mamba_prefill(p64, to_np(full), sh, scan="c")
    assert rel_l2(to_np(outs[rows]), ref["out"][:, L0:]) < TOL_BF16
    assert rel_l2(to_np(ss[rows]), ref["ssm_state"]) < TOL_BF16


@pytest.mark.parametrize("batch,L", [(3, 37), (2, 3), (4, 5), (1, 100), (2, 2)])
def test_prefill_conv_rows_through_x_proj(dev, batch, L):
    """The conv inside the bf16 in_proj epilogue, row by row: a warp holds 32
    token rows, so rows 0-2 of every 32-row slab whose window reaches the slab
    above are finished by a second kernel, and rows near a sequence start take
    their taps from the conv cache (random fp32 values here).  The x_proj
    output of the tensor-parallel first part is linear in the conv output, so
    each of its rows is compared with the oracle's on its own; short and
    ragged sequences put sequence starts at every lane position.  L = 2 takes
    the unfused path (fewer rows than the conv cache)."""
    sh = MambaShape(d_model=256, d_inner=256, dt_rank=16, dtype="bf16", inner_norm=False)
    mix, p64 = _mixer(sh, 21, dev, a_init="random")
    u = mamba_input(sh, batch, L, seed=21)
    g = torch.Generator().manual_seed(22)
    cs0 = torch.randn(batch, sh.d_inner, 3, generator=g)
    part, cs = mix.prefill_tp_begin(u.to(dev), conv_state_in=cs0.to(dev))
    ref = om.mamba_prefill(p64, to_np(u), sh, conv_state0=cs0.double().numpy(), keep=True)
    want = ref["proj"].reshape(batch * L, -1)
    got = to_np(part)
    row_err = np.linalg.norm(got - want, axis=1) / np.linalg.norm(want, axis=1)
    assert row_err.max() < 2e-2, (int(row_err.argmax()), float(row_err.max()))
    assert rel_l2(to_np(cs), ref["conv_state"]) < TOL_BF16


def test_bf16_prefill_long_unsplit_x_proj(dev):
    """20000 tokens at d_inner 512: x_proj has enough tiles to run without a
    k-split, and its sum + inner norms take the warp-per-token kernel
    (random norm weights, so each of the three segments is checked)."""
    sh = MambaShape(d_model=256, d_inner=512, dt_rank=32, dtype="bf16", inner_norm=True)
    mix, p64 = _mixer(sh, 31, dev, norm_init="random", a_init="random")
    u = mamba_input(sh, 1, 20000, seed=31)
    out, cs, ss = mix.prefill(u.to(dev))
    ref = om.mamba_prefill(p64, to_np(u), sh)
    assert rel_l2(to_np(out), ref["out"]) < TOL_BF16
    assert rel_l2(to_np(ss), ref["ssm_state"]) < TOL_BF16
    assert rel_l2(to_np(cs), ref["conv_state"]) < TOL_BF16
