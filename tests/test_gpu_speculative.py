"""Nested speculative decoding mechanics with one set of weights ("MatMamba: A Matryoshka State
Space Model", speculative-decoding paragraph): a small width drafts tokens with the recurrent step
from a saved state, and the full width verifies all of them with one prefill from that same saved
state, which is also the rollback point.  Acceptance rates need trained weights; what is checked
here is that each piece computes what the oracle computes, and that the draft leaves the saved
state untouched."""
import numpy as np
import pytest
import torch

from gpu_util import TOL, dims_of, ensure_built, make_block, max_abs_rel, to_device, to_np
from nested_mamba2_selective_b200 import matmamba_block_fwd, mm_device_status, ssd_step, synth

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS["decode_b256_1p4b"]


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


@pytest.fixture(scope="module")
def block():
    return make_block(W)


def test_draft_at_small_width_verify_at_full_width_from_saved_state(orc, block):
    wt, p64 = block
    dims = dims_of(W)
    b, L0, k = 2, 24, 5
    m_small, m_full = 512, 2048
    H, rows = dims.nheads, W.d_inner + 2 * W.d_state
    prompt = synth.activations((b, L0, W.d_model), "bf16", seed=340)
    drafts = synth.activations((b, k, W.d_model), "bf16", seed=341)

    # prompt at full width: the saved state is the rollback point
    s0 = torch.zeros((b, H, 64, 128), device="cuda")
    c0 = torch.zeros((b, rows, 3), device="cuda", dtype=torch.bfloat16)
    matmamba_block_fwd(wt, to_device(prompt, "bf16"), m_full, 256, ssm_state_out=s0, conv_state_out=c0)
    torch.cuda.synchronize()
    s0_keep, c0_keep = s0.clone(), c0.clone()

    # draft: k recurrent steps at the small width from a copy of the saved state
    s_d, c_d = s0.clone(), c0.clone()
    draft_out = [ssd_step(wt, s_d, c_d, to_device(drafts[:, i], "bf16"), m_small) for i in range(k)]
    # verify: one full-width prefill of the k drafted tokens from the saved state
    s_v = torch.zeros_like(s0)
    c_v = torch.zeros_like(c0)
    verify_out = matmamba_block_fwd(wt, to_device(drafts, "bf16"), m_full, 256, ssm_state_in=s0, conv_state_in=c0,
                                    ssm_state_out=s_v, conv_state_out=c_v)
    torch.cuda.synchronize()
    assert mm_device_status() == 0
    assert torch.equal(s0, s0_keep) and torch.equal(c0, c0_keep)  # the rollback point survives the draft

    # oracle: the same prompt prefill, the same k small-width steps, the same full-width verify
    s_ref = np.zeros((b, H, 64, 128))
    c_ref = np.zeros((b, rows, 3))
    orc.block_fwd(dims, p64, prompt, m_full, ssm_state_out=s_ref, conv_state_out=c_ref)
    s_dr, c_dr = s_ref.copy(), c_ref.copy()
    for i in range(k):
        ref_i = orc.block_step(dims, p64, drafts[:, i], m_small, s_dr, c_dr)
        assert max_abs_rel(to_np(draft_out[i]), ref_i) <= TOL["bf16"], i
    ref_full = orc.block_fwd(dims, p64, np.concatenate([prompt, drafts], axis=1), m_full)[:, L0:]
    assert max_abs_rel(to_np(verify_out), ref_full) <= TOL["bf16"]

    # accepting the first j drafts: resume from the full-width state after those j tokens, which
    # a prefill of drafts[:, :j] from the saved state gives
    j = 3
    s_j = torch.zeros_like(s0)
    c_j = torch.zeros_like(c0)
    matmamba_block_fwd(wt, to_device(drafts[:, :j], "bf16"), m_full, 256, ssm_state_in=s0, conv_state_in=c0,
                       ssm_state_out=s_j, conv_state_out=c_j)
    torch.cuda.synchronize()
    s_jr = np.zeros((b, H, 64, 128))
    c_jr = np.zeros((b, rows, 3))
    orc.block_fwd(dims, p64, np.concatenate([prompt, drafts[:, :j]], axis=1), m_full, ssm_state_out=s_jr,
                  conv_state_out=c_jr)
    assert max_abs_rel(to_np(s_j), s_jr) <= TOL["bf16"]
    assert max_abs_rel(to_np(c_j), c_jr) <= TOL["bf16"]
