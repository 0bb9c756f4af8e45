"""GPU parity of the GBLA layer (bat_gbla_forward, through the C ABI) against the fp64 oracle
(oracle/gbla.py), element by element, on bf16 inputs.

Bar, derived from the arithmetic.  y is stored in bf16 and its entries are not small: each row
has unit RMS before the gates, times g * silu(z), so |y| reaches ~15, where one bf16 rounding
alone is up to 2^-5.  The elementwise bound is therefore relative plus absolute:
|gpu - ref| <= 2e-2 + 1e-2 |ref|, from at most about 1 % accumulated relative error: the bf16
roundings of y (2^-9), of S and of phi(q~) (2^-9 each, entering o directly) and the fp16
roundings of the state operands w phi(k~) and v~ (2^-11 each; they do not simply average out
over the tokens: the RMS normalisation divides by the row's own output, so a row whose
weighted average nearly cancels magnifies them, which is why they are fp16 and not bf16), with
margin.  The aggregate bar is the attention path's: sum|gpu - ref| / sum|ref| <= 5e-3.

Ragged sequence lengths cover empty sequences, one token, tile multiples +-1 and several tiles
per chunk; guard rows around y must stay untouched; a long history (the bench workload's
length) is checked on sampled rows."""

import numpy as np
import pytest
import torch

import oracle.gbla as G
import prefix_shared_attention_b200 as bat
from workloads import gbla_tensors

pytestmark = pytest.mark.gpu

ABS, REL, MEAN_REL = 2e-2, 1e-2, 5e-3
GUARD = 64


def make_inputs(lens, H, seed, device="cpu"):
    return gbla_tensors(lens, H, seed, device=device)


def run_gpu(x, so, H, num_sms=0):
    xd = {k: v.cuda().contiguous() for k, v in x.items()}
    T = xd["q"].shape[0]
    buf = torch.full((T + 2 * GUARD, H, 128), -7.25, dtype=torch.bfloat16, device="cuda")
    buf[GUARD:GUARD + T] = float("nan")
    y = buf[GUARD:GUARD + T]
    with bat.GblaPlan(so, H, num_sms=num_sms) as plan:
        bat.bat_gbla_forward(plan, xd["q"], xd["k"], xd["v"], xd["a"], xd["z"], xd["cq"], xd["ck"], xd["cv"], xd["g"], y=y)
        st = bat.bat_get_device_status()
    assert st == bat.BAT_OK, bat.last_error()
    assert bool((buf[:GUARD] == -7.25).all()) and bool((buf[GUARD + T:] == -7.25).all()), "write outside y"
    return y


def oracle_y(x, so, rows=None):
    return G.gbla_forward(x["q"], x["k"], x["v"], x["a"], x["z"], x["cq"], x["ck"], x["cv"], x["g"], so, rows)


def check(got, ref, what):
    got = np.asarray(got, np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite or unwritten rows"
    d = np.abs(got - ref)
    excess = float((d - (ABS + REL * np.abs(ref))).max())
    mr = float(d.sum() / np.abs(ref).sum())
    worst = float((d / (ABS + REL * np.abs(ref))).max())
    assert excess <= 0 and mr <= MEAN_REL, (f"{what}: max-abs {d.max():.3g}, worst ratio to the bound {worst:.3g}, "
                                            f"mean-rel {mr:.3g}")
    return worst, mr


@pytest.mark.parametrize("lens,H,num_sms", [
    ([1, 3, 127, 128, 129, 300, 0, 517], 2, 0),
    ([700, 1, 256, 383], 3, 4),            # few SMs: several tiles per chunk
    ([5000], 1, 0),
])
def test_gbla_matches_oracle(lens, H, num_sms):
    x, so = make_inputs(lens, H, seed=len(lens) + H)
    y = run_gpu(x, so, H, num_sms)
    check(y.float().cpu().numpy(), oracle_y(x, so), f"lens={lens}")


def test_gbla_gate_closed_tokens_are_forgotten():
    """Soft forgetting on the GPU: tokens whose gate logit is very negative change nothing for
    the other tokens (compared with the oracle of the same inputs, where they weigh ~0)."""
    lens = [400]
    x, so = make_inputs(lens, 2, seed=9)
    x["a"][100:300] = -30.0
    y = run_gpu(x, so, 2)
    check(y.float().cpu().numpy(), oracle_y(x, so), "closed gates")


@pytest.mark.parametrize("shift", [-20.0, -30.0])
def test_gbla_nearly_closed_gates_everywhere(shift):
    """Every key gate nearly closed (logits N(shift, 2^2): w ~ 1e-9 .. 1e-13).  The gates cancel
    between numerator and denominator (n.phi(q~) still dwarfs the 1e-6), so the output is an
    ordinary weighted average of normal magnitude; the gated keys must not vanish in the
    operands' range on the way."""
    lens, H = [3000, 700], 2
    x, so = make_inputs(lens, H, seed=31)
    x["a"] = (x["a"].float() + shift).to(torch.bfloat16)
    y = run_gpu(x, so, H)
    ref = oracle_y(x, so)
    assert np.abs(ref).max() > 1.0, "the case must have outputs of normal magnitude"
    check(y.float().cpu().numpy(), ref, f"gates shifted by {shift}")


def test_gbla_long_history_sampled():
    """The bench workload's shape for one sequence: a 32768-token history (H = 8), checked on
    256 sampled rows of every head."""
    lens, H = [32768], 8
    x, so = make_inputs(lens, H, seed=77)
    y = run_gpu(x, so, H)
    rows = np.sort(np.random.default_rng(5).choice(so[-1], 256, replace=False))
    ref = oracle_y(x, so, rows)
    check(y.float().cpu().numpy()[rows], ref, "long history")


def test_gbla_wait_timeout_reports_and_context_survives():
    """Failure detection on the GBLA kernels: with a 1 ns wait limit the first wait whose phase
    has not completed (a tile that has not landed yet) runs out, the kernels abort (their copies
    and MMAs in flight drained, tensor memory freed), the status word reports BAT_ERR_TIMEOUT,
    and the next run on the same context is correct."""
    lens, H = [3000, 2000], 2
    x, so = make_inputs(lens, H, seed=21)
    xd = {k: v.cuda().contiguous() for k, v in x.items()}
    bat.bat_set_wait_timeout_ns(1)
    try:
        with bat.GblaPlan(so, H) as plan:
            y = torch.empty_like(xd["q"])
            bat.bat_gbla_forward(plan, xd["q"], xd["k"], xd["v"], xd["a"], xd["z"], xd["cq"], xd["ck"], xd["cv"], xd["g"],
                                 y=y)
            st = bat.bat_get_device_status()
    finally:
        bat.bat_set_wait_timeout_ns(0)
    assert st == bat.BAT_ERR_TIMEOUT, f"expected BAT_ERR_TIMEOUT, got {st}: {bat.last_error()}"
    y = run_gpu(x, so, H)
    check(y.float().cpu().numpy(), oracle_y(x, so), "after a timed-out run")
    assert bat.bat_get_device_status() == bat.BAT_OK
