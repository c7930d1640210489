"""The give-up path of the library's bounded waits, made to run out on purpose.

Every mbarrier wait in the kernels stops after a fixed number of unsuccessful
polls, sets the workspace error word to ASM_ERR_TIMEOUT and lets its CTA
finish.  asm_wait_selftest runs that path on a barrier nothing arrives at (no
copy in flight, no tensor memory held); the host then reads the error word,
and the context must still run the library's kernels correctly.
"""
import pytest
import torch

from long_prefix_attention_b200 import ops

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_reports_timeout_and_leaves_the_context_usable():
    ws = ops.alloc_workspace(256, "cuda")
    # a short probe first: it bounds what the library's own wait will take
    probe_polls = 4096
    ns_probe = ops.asm_wait_selftest(probe_polls, ws)
    assert ops.asm_workspace_error(ws) == ops.ASM_ERR_TIMEOUT
    limit = ops.asm_wait_spin_limit()
    estimate_s = ns_probe * (limit / probe_polls) / 1e9
    print(f"probe: {probe_polls} polls in {ns_probe / 1e3:.1f} us; the library's {limit} polls: ~{estimate_s:.2f} s")
    assert estimate_s < 5.0, f"a library wait would take about {estimate_s:.1f} s before giving up"

    # the library's own bounded wait
    ops.asm_workspace_init(ws)
    assert ops.asm_workspace_error(ws) == 0
    ns_full = ops.asm_wait_selftest(0, ws)
    print(f"library wait gave up after {ns_full / 1e9:.3f} s")
    assert ops.asm_workspace_error(ws) == ops.ASM_ERR_TIMEOUT
    assert 0 < ns_full < 10e9

    # the context still works: merging with the empty state leaves a state unchanged
    g = torch.Generator(device="cuda").manual_seed(3)
    a = torch.randn(64, 128, device="cuda", generator=g).to(torch.bfloat16)
    z = torch.randn(64, device="cuda", generator=g)
    a0, z0 = a.clone(), z.clone()
    ops.asm_merge_states(a, z, torch.zeros_like(a), torch.full_like(z, float("-inf")))
    torch.cuda.synchronize()
    assert torch.equal(a, a0) and torch.equal(z, z0)


def test_selftest_rejects_bad_arguments():
    ws = ops.alloc_workspace(256, "cuda")
    with pytest.raises(ops.AsmError):
        ops.asm_wait_selftest(-1, ws)
    with pytest.raises(ops.AsmError):
        ops.asm_wait_selftest(16, ws[:16])
