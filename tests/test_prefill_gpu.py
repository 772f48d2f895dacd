"""kda_chunk_fwd (CUDA, through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

from gated_delta_rule_100_b200 import inputs, kda
from kda_testlib import assert_close, f64, oracle_prefill

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(autouse=True)
def _reset_hooks():
    kda.inject_timeout(0)
    kda.set_wait_limit(0)
    kda.force_exact(False)
    kda.block_refs(False)
    yield
    kda.inject_timeout(0)
    kda.set_wait_limit(0)
    kda.force_exact(False)
    kda.block_refs(False)
    assert kda.stream_status() == kda.KDA_OK


def run(d, scale, **kw):
    out, hT = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], scale, d["h0"], **kw)
    torch.cuda.synchronize()
    return out, hT


def check(d, scale, what, **kw):
    out, hT = run(d, scale, **kw)
    o_ref, s_ref = oracle_prefill(d, scale)
    assert_close(f64(out), o_ref, f"{what} out")
    assert_close(f64(hT), s_ref, f"{what} hT")
    return out, hT


@pytest.mark.parametrize("name", ["oracle_scale_B1_H1_T256_d64", "prefill_B1_H4_T2048_d128"])
def test_config_full(name):
    cfg = inputs.CONFIGS[name]
    d = inputs.make_config(cfg, device=DEV)
    check(d, cfg.scale, name)


@pytest.mark.parametrize("T", [1, 15, 63, 64, 65, 129, 1000])
def test_ragged_lengths(T):
    d = inputs.make_prefill(2, T, 3, 128, 128, decay=0.05, h0_std=0.02, seed=100 + T, device=DEV)
    check(d, 128 ** -0.5, f"T={T}")


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64), (128, 128)])
def test_head_dims(dk, dv):
    d = inputs.make_prefill(1, 300, 2, dk, dv, decay=0.1, h0_std=0.02, seed=7, device=DEV)
    check(d, dk ** -0.5, f"dk={dk} dv={dv}")


def test_value_slices_are_independent():
    """The columns of the state evolve independently (each chain CTA carries a
    slice of them), so the first 64 columns of a dv = 128 run must equal, bit
    for bit, a dv = 64 run on those columns alone."""
    d = inputs.make_prefill(2, 200, 2, 128, 128, decay=0.05, h0_std=0.02, seed=8, device=DEV)
    out, hT = check(d, 0.1, "dv=128")
    half = dict(d)
    half["v"] = d["v"][..., :64].contiguous()
    half["h0"] = d["h0"][..., :64].contiguous()
    out2, hT2 = run(half, 0.1)
    assert torch.equal(out2, out[..., :64])
    assert torch.equal(hT2, hT[..., :64])


def test_null_h0_and_null_hT():
    d = inputs.make_prefill(1, 130, 2, 128, 128, decay=0.05, h0_std=0.0, seed=9, device=DEV)
    out, hT = run(d, 0.2, final_state=False)
    assert hT is None
    o_ref, _ = oracle_prefill(d, 0.2)
    assert_close(f64(out), o_ref, "hT=NULL out")


def test_h0_aliases_hT():
    d = inputs.make_prefill(2, 150, 2, 128, 128, decay=0.05, h0_std=0.02, seed=10, device=DEV)
    o_ref, s_ref = oracle_prefill(d, 0.3)
    state = d["h0"].clone()
    out, hT = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], 0.3, state, hT=state)
    torch.cuda.synchronize()
    assert hT.data_ptr() == state.data_ptr()
    assert_close(f64(out), o_ref, "aliased out")
    assert_close(f64(state), s_ref, "aliased state")


def test_zero_length():
    d = inputs.make_prefill(1, 0, 2, 64, 64, decay=0.05, h0_std=0.02, seed=11, device=DEV)
    out, hT = run(d, 0.3)
    assert out.shape[1] == 0
    assert torch.equal(hT, d["h0"])


def test_beta_zero_closed_form():
    """beta = 0: the state only decays, S_t = Diag(e^{Gamma_t}) h0."""
    d = inputs.make_prefill(1, 333, 2, 128, 128, decay=0.1, h0_std=0.5, seed=12, device=DEV)
    d["beta"].zero_()
    out, hT = run(d, 0.25)
    g = f64(d["g"])
    Gam = np.cumsum(g, axis=1)
    h0 = f64(d["h0"])
    want = 0.25 * np.einsum("bthc,bhcd->bthd", np.exp(Gam) * f64(d["q"]), h0)
    assert_close(f64(out), want, "beta=0 out")
    assert_close(f64(hT), np.exp(Gam[:, -1])[..., None] * h0, "beta=0 hT")


def test_beta_one_write_then_read():
    """beta = 1 and q = k: reading right after the write returns |k|^2-weighted v
    (S_t^T k_t = (1-|k|^2)(D S)^T k + |k|^2 v); checked against the oracle."""
    d = inputs.make_prefill(1, 200, 2, 128, 128, decay=0.05, h0_std=0.02, seed=13, device=DEV)
    d["beta"].fill_(1.0)
    d["q"] = d["k"].clone()
    check(d, 1.0, "beta=1 q=k")


@pytest.mark.parametrize("decay", [0.0, 5.0])
def test_decay_extremes(decay):
    """g = 0 (no decay) and g = -5 softplus(N(0,1)) (fast forgetting)."""
    d = inputs.make_prefill(1, 500, 2, 128, 128, decay=decay, h0_std=0.02, seed=14, device=DEV)
    check(d, 128 ** -0.5, f"decay={decay}")


def test_continuation():
    """chunk_fwd(T1) then chunk_fwd(T2) from its hT equals the oracle over T1 + T2
    (the split is not on a chunk boundary)."""
    d = inputs.make_prefill(1, 400, 2, 128, 128, decay=0.05, h0_std=0.02, seed=15, device=DEV)
    cut = 136
    a = {k: (v[:, :cut].contiguous() if k != "h0" else v) for k, v in d.items()}
    o1, s1 = run(a, 0.2)
    b = {k: (v[:, cut:].contiguous() if k != "h0" else s1) for k, v in d.items()}
    o2, s2 = run(b, 0.2)
    o_ref, s_ref = oracle_prefill(d, 0.2)
    assert_close(f64(torch.cat([o1, o2], dim=1)), o_ref, "continuation out")
    assert_close(f64(s2), s_ref, "continuation hT")


def test_value_column_permutation():
    d = inputs.make_prefill(1, 180, 2, 128, 128, decay=0.05, h0_std=0.02, seed=16, device=DEV)
    out, hT = run(d, 0.2)
    perm = torch.randperm(128, generator=torch.Generator().manual_seed(0)).to(DEV)
    dp = dict(d)
    dp["v"] = d["v"][..., perm].contiguous()
    dp["h0"] = d["h0"][..., perm].contiguous()
    out_p, hT_p = run(dp, 0.2)
    o_ref, s_ref = oracle_prefill(dp, 0.2)
    assert_close(f64(out_p), o_ref, "permuted out")
    assert_close(f64(hT_p), s_ref, "permuted hT")
    assert_close(f64(out_p), f64(out[..., perm]), "permuted vs unpermuted out")


def test_timeout_path_reports_and_recovers():
    """The fault-injection hook makes every CTA wait on a barrier nothing signals:
    the bounded wait must give up, the kernel must record KDA_ERR_TIMEOUT,
    release what it holds and return; the next call must be correct."""
    d = inputs.make_prefill(1, 256, 2, 128, 128, decay=0.05, h0_std=0.02, seed=17, device=DEV)
    kda.inject_timeout(1000)
    run(d, 0.2)
    assert kda.stream_status() == kda.KDA_ERR_TIMEOUT
    kda.inject_timeout(0)
    check(d, 0.2, "after timeout")


def test_training_shape_full():
    cfg = inputs.CONFIGS["training_B8_H32_T4096_d128"]
    d = inputs.make_config(cfg, device=DEV)
    out, hT = run(d, cfg.scale)
    o_ref, s_ref = oracle_prefill(d, cfg.scale)
    assert_close(f64(out), o_ref, "training out")
    assert_close(f64(hT), s_ref, "training hT")


def test_long_context_sampled():
    """Full 1M-token launch; the oracle checks heads 0-1 over the first 65,536
    tokens and head 0's final state over all tokens."""
    cfg = inputs.CONFIGS["long_context_B1_H32_T1M_d128"]
    d = inputs.make_config(cfg, device=DEV)
    out, hT = run(d, cfg.scale)
    o_ref, _ = oracle_prefill(d, cfg.scale, heads=slice(0, 2), tokens=65536)
    assert_close(f64(out[:, :65536, 0:2]), o_ref, "long-context out (heads 0-1, 64k tokens)")
    _, s_ref = oracle_prefill(d, cfg.scale, heads=slice(0, 1))
    assert_close(f64(hT[:, 0:1]), s_ref, "long-context hT (head 0)")


def steep_gate(d, pattern):
    """Decays far beyond the workloads': every chunk (constant -12), isolated
    spikes (-30 on every 7th token), or one burst of four -25 tokens inside the
    second half of a 16-token block (one steep chunk among ordinary ones)."""
    g = d["g"]
    if pattern == "const_m12":
        g.fill_(-12.0)
    elif pattern == "every7_m30":
        g[:, 6::7] = -30.0
    elif pattern == "burst_m25":
        g[:, 41:45] = -25.0
    return d


@pytest.mark.parametrize("gate", ["per_channel", "scalar"])
@pytest.mark.parametrize("pattern", ["const_m12", "every7_m30", "burst_m25"])
@pytest.mark.parametrize("T", [64, 1000])
def test_steep_decay(T, pattern, gate):
    """Any finite g <= 0: chunks whose decay would push a split factor past e^80
    take the exact path; the result must match the oracle either way, on both
    gate forms (the scalar gate is channel 0 of the gate, broadcast for the oracle)."""
    d = steep_gate(inputs.make_prefill(1, T, 2, 128, 128, decay=0.05, h0_std=0.02, seed=500 + T, device=DEV),
                   pattern)
    scale = 128 ** -0.5
    if gate == "scalar":
        gs = d["g"][..., 0].contiguous()
        d["g"] = gs.unsqueeze(-1).expand_as(d["g"]).contiguous()
        out, hT = kda.gdn_chunk_fwd(d["q"], d["k"], d["v"], gs, d["beta"], scale, d["h0"])
    else:
        out, hT = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], scale, d["h0"])
    torch.cuda.synchronize()
    o_ref, s_ref = oracle_prefill(d, scale)
    assert_close(f64(out), o_ref, f"{pattern} T={T} {gate} out")
    assert_close(f64(hT), s_ref, f"{pattern} T={T} {gate} hT")


@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128)])
def test_exact_path_matches_fast_path(dk, dv):
    """The exact path (forced on every chunk) and the tensor-core path agree with
    the oracle and with each other on ordinary inputs."""
    d = inputs.make_prefill(2, 300, 2, dk, dv, decay=0.1, h0_std=0.02, seed=600 + dk, device=DEV)
    fast_o, fast_s = check(d, dk ** -0.5, f"fast path dk={dk}")
    kda.force_exact(True)
    ex_o, ex_s = check(d, dk ** -0.5, f"exact path dk={dk}")
    kda.force_exact(False)
    assert_close(f64(ex_o), f64(fast_o), "exact vs fast out")
    assert_close(f64(ex_s), f64(fast_s), "exact vs fast hT")


@pytest.mark.parametrize("dk,dv", [(64, 128), (128, 64), (128, 128)])
@pytest.mark.parametrize("T", [77, 1000])
def test_mild_and_block_forms_agree(T, dk, dv):
    """A chunk whose decay is mild (every key channel keeps e^{Gamma_C} >= e^-40) is
    formed with one reference at its start; the 16-token block references (the
    form of chunks with stronger decay, forced here on every chunk) must give the
    same results: both match the oracle and each other."""
    d = inputs.make_prefill(2, T, 2, dk, dv, decay=0.1, h0_std=0.02, seed=650 + T + dk, device=DEV)
    scale = dk ** -0.5
    mild_o, mild_s = check(d, scale, f"mild form T={T} {dk}x{dv}")
    kda.block_refs(True)
    blk_o, blk_s = check(d, scale, f"block form T={T} {dk}x{dv}")
    kda.block_refs(False)
    assert_close(f64(blk_o), f64(mild_o), "block vs mild form out")
    assert_close(f64(blk_s), f64(mild_s), "block vs mild form hT")


@pytest.mark.parametrize("gate", ["per_channel", "scalar"])
def test_decay_around_the_mild_limit(gate):
    """Chunks on both sides of the mild limit in one sequence: in each chunk one key
    channel (channel 0 for the scalar gate) decays at a constant rate whose chunk
    total ranges from -30 to -70 (mild below 40, block references above, no
    16-token block steep), the others at the workload's rate; the tail chunk is
    ragged.  Every chunk must match the oracle whichever form it took."""
    T = 16 * 64 + 23
    d = inputs.make_prefill(1, T, 2, 128, 128, decay=0.05, h0_std=0.02, seed=660, device=DEV)
    g = d["g"]
    rates = torch.linspace(30.0, 70.0, (T + 63) // 64, device=DEV) / 64.0
    ch = 0 if gate == "scalar" else 37
    for n, r in enumerate(rates.tolist()):
        g[0, 64 * n:64 * (n + 1), :, ch] = -r
    scale = 128 ** -0.5
    if gate == "scalar":
        gs = g[..., 0].contiguous()
        d["g"] = gs.unsqueeze(-1).expand_as(g).contiguous()
        out, hT = kda.gdn_chunk_fwd(d["q"], d["k"], d["v"], gs, d["beta"], scale, d["h0"])
    else:
        out, hT = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], scale, d["h0"])
    torch.cuda.synchronize()
    o_ref, s_ref = oracle_prefill(d, scale)
    assert_close(f64(out), o_ref, f"mild limit {gate} out")
    assert_close(f64(hT), s_ref, f"mild limit {gate} hT")


def test_large_values_and_state():
    """|v| ~ 100 and h0 ~ N(0, 1): the fp16 operands (P, decayed keys, corrected
    values) stay in range.  The method is linear in (v, h0), so this is the base
    problem scaled by ~100: rel-L2 keeps its bar and the max-abs bar scales by 100."""
    d = inputs.make_prefill(2, 1000, 2, 128, 128, decay=0.05, h0_std=1.0, seed=700, device=DEV)
    d["v"] = (d["v"].float() * 100.0).to(torch.bfloat16)
    out, hT = run(d, 128 ** -0.5)
    o_ref, s_ref = oracle_prefill(d, 128 ** -0.5)
    assert_close(f64(out), o_ref, "|v|~100 out", mabs=100 * 2e-2)
    assert_close(f64(hT), s_ref, "|v|~100 hT", mabs=100 * 2e-2)


@pytest.mark.parametrize("pieces", [(16,), (32,), (1, 17, 50, 64, 23)])
def test_chunk_boundaries_do_not_matter(pieces):
    """The chunkwise form equals the recurrence whatever the blocking.  Feeding the
    same sequence through chunk_fwd in pieces (state carried through hT -> h0) puts
    the chunk boundaries every 16 or 32 tokens (chunk sizes 16 and 32 of the same
    kernels: each call holds one partial chunk) or at irregular offsets; all must
    match one whole-sequence call (chunk size 64) and the oracle."""
    T = 448
    d = inputs.make_prefill(1, T, 2, 128, 128, decay=0.1, h0_std=0.02, seed=800, device=DEV)
    whole_o, whole_s = check(d, 0.2, "whole sequence")
    outs, state, t0, n = [], d["h0"], 0, 0
    while t0 < T:
        L = min(pieces[n % len(pieces)], T - t0)
        part = {k: (v[:, t0:t0 + L].contiguous() if k != "h0" else state) for k, v in d.items()}
        o, state = run(part, 0.2)
        outs.append(o)
        t0, n = t0 + L, n + 1
    o_ref, s_ref = oracle_prefill(d, 0.2)
    pieced = torch.cat(outs, dim=1)
    assert_close(f64(pieced), o_ref, f"pieces {pieces} out")
    assert_close(f64(state), s_ref, f"pieces {pieces} hT")
    assert_close(f64(pieced), f64(whole_o), f"pieces {pieces} vs whole out")
    assert_close(f64(state), f64(whole_s), f"pieces {pieces} vs whole hT")


def test_kernel_timing_hook_stamps_every_launch():
    """The measurement hook: every prefill launch stamps its busy interval; each
    kind's summed time is positive and within the call's wall time on the device."""
    d = inputs.make_prefill(2, 2000, 4, 128, 128, decay=0.05, h0_std=0.02, seed=18, device=DEV)
    run(d, 0.1)
    kda.kernel_times()  # forget anything recorded before
    kda.kernel_timing(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    run(d, 0.1)
    e1.record()
    torch.cuda.synchronize()
    kda.kernel_timing(False)
    t = kda.kernel_times()
    wall = e0.elapsed_time(e1)
    assert t["prep"][1] >= 1 and t["chain"][1] >= 1 and t["exact"][1] >= 1
    for kind in ("prep", "chain"):
        assert 0.0 < t[kind][0] <= wall * 1.05 + 0.01, (kind, t[kind], wall)
    assert kda.kernel_times() == {k: (0.0, 0) for k in kda.KERNEL_KINDS}  # read once


def test_kernel_launch_timeline():
    """The hook's per-launch form: one entry per launch in launch order, each with
    start <= end; prep precedes the chain it feeds, and the list is read once."""
    d = inputs.make_prefill(1, 3000, 2, 128, 128, decay=0.05, seed=19, device=DEV)
    run(d, 0.1)
    kda.kernel_launches()
    kda.kernel_timing(True)
    run(d, 0.1)
    torch.cuda.synchronize()
    kda.kernel_timing(False)
    L = kda.kernel_launches()
    kinds = [k for k, _, _ in L]
    assert kinds[:2] == ["prep", "exact"] and "chain" in kinds, kinds
    assert all(e >= s for _, s, e in L), L
    p = next(x for x in L if x[0] == "prep")
    c = next(x for x in L if x[0] == "chain")
    assert c[1] >= p[2] - 1e-6  # the chain starts after its records are written
    assert kda.kernel_launches() == []


@pytest.mark.parametrize("B,H,T", [(64, 32, 100), (256, 16, 1)])
def test_many_heads_short_sequences(B, H, T):
    """Thousands of (b, h) with one or two chunks each: one chain CTA per (b, h)
    (many waves), a partial chunk, h0 read and hT written per (b, h).  Checked
    against the oracle on every sequence of two heads and on all heads of two
    batch rows."""
    d = inputs.make_prefill(B, T, H, 128, 128, decay=0.05, h0_std=0.02, seed=23 + T, device=DEV)
    out, hT = run(d, 128 ** -0.5)
    assert kda.stream_status() == kda.KDA_OK
    o_ref, s_ref = oracle_prefill(d, 128 ** -0.5, heads=[0, H - 1])
    assert_close(f64(out[:, :, [0, H - 1]]), o_ref, f"B{B} H{H} T{T} out (heads 0, {H - 1})")
    assert_close(f64(hT[:, [0, H - 1]]), s_ref, f"B{B} H{H} T{T} hT (heads 0, {H - 1})")
    o_ref, s_ref = oracle_prefill(d, 128 ** -0.5, batches=[0, B - 1])
    assert_close(f64(out[[0, B - 1]]), o_ref, f"B{B} H{H} T{T} out (batches 0, {B - 1})")
    assert_close(f64(hT[[0, B - 1]]), s_ref, f"B{B} H{H} T{T} hT (batches 0, {B - 1})")
