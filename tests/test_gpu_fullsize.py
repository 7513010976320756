"""GPU parity at the full model sizes, in the launch configuration the
benchmark times (the library picks the persistent grid from the SM count and
occupancy).  The 130M list is compared completely; the 1.1B and 2.7B lists on
sampled blocks (first, last and random blocks of every quantised tensor, more
on the LM head) plus every fp32-state tensor.  Blocks are independent and
every draw is keyed by (seed, step, tensor, element), so a sampled block's
oracle result is exactly the full run's.  Inputs come from the seeded device
generator; the oracle's copies are taken before any step runs."""
import numpy as np
import pytest

import oracle
import workloads
from gpu_common import assert_state_equal, assert_weights_close, binding, oracle_for, sampled_parity

pytestmark = pytest.mark.gpu


def test_gpt_130m_one_step_prewarmed_zipsr():
    """GPT-2-style 130M list, one step at t = 1000 from pre-warmed synthetic
    state, ZIP-SR; every element of every tensor compared."""
    import torch
    name = "gpt-130m"
    ts = workloads.tensor_list(name)
    params, grads = workloads.device_inputs(name, ts)
    blob = workloads.synthetic_state_blob(ts, 0, 999, is_fp32=oracle.is_fp32_state)
    ws = [p.cpu().numpy().copy() for p in params]
    gs = [g.view(torch.int16).cpu().numpy().view(np.uint16).copy() for g in grads]
    B = binding()
    opt = B.AdamW4(params, grads, ts, lr=1e-3, vcode=0, seed=0)
    try:
        opt.load_state_blob(blob)
        assert opt.t == 999
        opt.step()
        torch.cuda.synchronize()
        ref = oracle_for(ts, vcode=0)
        ref.import_state(blob)
        old = [w.copy() for w in ws]
        ref.step(ws, gs)
        for i, p in enumerate(params):
            assert_weights_close(p.cpu().numpy(), ws[i], old[i], f"{name} tensor {i}")
        assert_state_equal(opt.state_dict_blob(), ref.export_state(), 0, name)
    finally:
        opt.close()
        del params, grads
        torch.cuda.empty_cache()


def test_llama_1p1b_zeeden_lm_head_phase_sampled():
    """Llama-style 1.1B list, ZE-EDEN, ten steps t = 901..910 of a 1000-step
    run (the LM head's m is rounded stochastically), pre-warmed state."""
    n = sampled_parity("llama-1.1b", vcode=1, steps=10, t0=900, total_steps=1000, prewarm=True,
                       what="llama-1.1b")
    assert n > 1000


@pytest.mark.parametrize("vcode", [0, 1, 2, 3, 4, 5])
def test_gpt_2p7b_sampled(vcode):
    """GPT-style 2.7B list (the benchmark workload), two steps from zero state,
    for the two methods and the three state-space variants."""
    n = sampled_parity("gpt-2.7b", vcode=vcode, steps=2, t0=0, what=f"gpt-2.7b v{vcode}")
    assert n > 1500


def test_tensor_past_2_31_elements():
    """One 4-bit tensor of 2^31 + 300 values (element offsets and pointer
    arithmetic past 32 bits, a ragged tail), with an LM head in its final-10%
    phase and a norm tensor beside it; ZIP-SR, two steps, sampled blocks
    including the two around element 2^31."""
    n = sampled_parity("huge-2g", vcode=0, steps=2, t0=8, total_steps=10, what="huge-2g")
    assert n > 100


@pytest.mark.parametrize("vcode", [0, 1])
def test_gpt_2p7b_step_100_teacher_forced(vcode):
    """The benchmark's run length: 99 steps of the 2.7B list on the GPU (one
    seeded grad set reused, as the benchmark times it), then step 100
    teacher-forced -- the oracle starts from the GPU's state and weights after
    step 99 and computes step 100 on sampled blocks and every fp32-state
    tensor.  By then v has settled near g^2.  Reports the share of sampled v
    codes at 0 after step 99: for ZIP-SR that is the zero code point, which
    preconditioner-space rounding picks from the first cell only with
    probability about eps / sqrt(v_hat), v_hat = v / (1 - b2^t) ("ZIP-SR
    4-bit AdamW -- Preconditioner-space stochastic rounding", worked example
    paragraph), so it stays rare while v is well above eps^2, and the values
    of that cell land on code 1, its upper point (also reported); for
    ZE-EDEN code 0 is the lowest nonzero point 1/16."""
    from gpu_common import teacher_forced_parity
    n, zero_share, one_share = teacher_forced_parity("gpt-2.7b", vcode, 100,
                                                     what=f"gpt-2.7b v{vcode} t100")
    assert n > 1500
    assert 0.0 <= zero_share <= 1.0 and 0.0 <= one_share <= 1.0
    print(f"v{vcode}: {n} blocks checked at step 100; v codes at 0 after step 99: "
          f"{100 * zero_share:.3f}%, at 1: {100 * one_share:.3f}%")


@pytest.mark.parametrize("vcode", [0, 1])
def test_gpt_130m_step_1000_teacher_forced_lm_head_phase(vcode):
    """A longer run on the 130M list: 999 GPU steps (one grad set reused), then
    step 1000 teacher-forced against the oracle, with total_steps = 1000 so
    that steps past 900 are in the LM head's final-10% phase ("ZIP-SR 4-bit
    AdamW -- Preconditioner-space stochastic rounding", ZE-EDEN paragraph):
    the tied embedding's m is then rounded stochastically on the NF4 grid,
    and the oracle checks extra blocks of it."""
    from gpu_common import teacher_forced_parity
    n, zero_share, one_share = teacher_forced_parity(
        "gpt-130m", vcode, 1000, what=f"gpt-130m v{vcode} t1000", total_steps=1000)
    assert n > 300
    print(f"v{vcode}: {n} blocks checked at step 1000; v codes at 0 after step 999: "
          f"{100 * zero_share:.3f}%, at 1: {100 * one_share:.3f}%")
