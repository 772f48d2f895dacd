"""The two-level (segment-parallel) state pass of kda_chunk_fwd: parts of a
segment formed in parallel (zero-start states and dk x dk transitions), a
sequential fix-up of the parts' start states, then every part's outputs in
parallel.  Against the fp64 oracle and against the plain pass."""
import pytest
import torch

from gated_delta_rule_100_b200 import inputs, kda
from kda_testlib import assert_close, f64, oracle_prefill

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(autouse=True)
def _reset_hooks():
    kda.set_parts(0)
    kda.set_record_cap(0)
    yield
    kda.set_parts(0)
    kda.set_record_cap(0)
    assert kda.stream_status() == kda.KDA_OK


def run(d, scale, **kw):
    out, hT = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], scale, d["h0"], **kw)
    torch.cuda.synchronize()
    return out, hT


@pytest.mark.parametrize("parts", [3, 5, 8])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 64)])
def test_two_level_matches_oracle_and_plain(parts, dk, dv):
    """T = 3000 (47 chunks) with h0 != 0, cut into 3, 5 or 8 parts."""
    d = inputs.make_prefill(1, 3000, 2, dk, dv, decay=0.05, h0_std=0.02, seed=1400 + parts, device=DEV)
    scale = dk ** -0.5
    kda.set_parts(1)
    plain_o, plain_s = run(d, scale)
    kda.set_parts(parts)
    out, hT = run(d, scale)
    o_ref, s_ref = oracle_prefill(d, scale)
    assert_close(f64(out), o_ref, f"two-level P={parts} {dk}x{dv} out")
    assert_close(f64(hT), s_ref, f"two-level P={parts} {dk}x{dv} hT")
    assert_close(f64(out), f64(plain_o), f"two-level vs plain P={parts} out")
    assert_close(f64(hT), f64(plain_s), f"two-level vs plain P={parts} hT")


def test_two_level_across_segments():
    """Parts inside each of several segments (record cap of 3 x 16 chunks on two
    buffers), the state carried between segments; no final state wanted too."""
    d = inputs.make_prefill(1, 6000, 2, 128, 128, decay=0.05, h0_std=0.02, seed=1500, device=DEV)
    kda.set_record_cap(2 * 2 * 16 * 74240)  # segments of 16 chunks, 6 segments
    kda.set_parts(4)
    out, hT = run(d, 0.1)
    out2, _ = run(d, 0.1, final_state=False)
    o_ref, s_ref = oracle_prefill(d, 0.1)
    assert_close(f64(out), o_ref, "two-level segmented out")
    assert_close(f64(hT), s_ref, "two-level segmented hT")
    assert torch.equal(out, out2)


def test_two_level_automatic_few_heads():
    """Automatic choice on a long sequence with few heads (B1 H2 T16384: 256 chunks)."""
    d = inputs.make_prefill(1, 16384, 2, 128, 128, decay=0.02, h0_std=0.02, seed=1600, device=DEV)
    out, hT = run(d, 128 ** -0.5)
    o_ref, s_ref = oracle_prefill(d, 128 ** -0.5)
    assert_close(f64(out), o_ref, "automatic two-level out")
    assert_close(f64(hT), s_ref, "automatic two-level hT")


def test_two_level_steep_decay_and_aliasing():
    """Steep chunks (exact path) inside parts, and h0 == hT aliasing."""
    d = inputs.make_prefill(1, 2000, 2, 128, 128, decay=0.05, h0_std=0.02, seed=1700, device=DEV)
    d["g"][:, 500:520] = -30.0
    o_ref, s_ref = oracle_prefill(d, 0.1)
    kda.set_parts(5)
    state = d["h0"].clone()
    out, hT = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], 0.1, state, hT=state)
    torch.cuda.synchronize()
    assert_close(f64(out), o_ref, "two-level steep out")
    assert_close(f64(state), s_ref, "two-level steep hT (aliased)")
