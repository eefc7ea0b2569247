"""The allocation-free attention backward (gpt2_op_attention_bwd_noalloc).

Some callers may not allocate device memory (their framework's allocator or a
fixed budget owns it all); this entry point keeps its scratch in a fixed device
array instead. It must give the same gradients as gpt2_op_attention_bwd, call
after call, through the C ABI. This file is collected last on purpose.
"""
import pytest
import torch

import train_step_b200 as tsb

pytestmark = pytest.mark.gpu


def _inputs(B, T, NH, hd, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    C = NH * hd
    qkv = torch.randn(B * T, 3 * C, generator=g).to(dtype).cuda()
    dout = torch.randn(B * T, C, generator=g).to(dtype).cuda()
    out = torch.zeros(B * T, C, dtype=dtype, device="cuda")
    lse = torch.zeros(B, NH, T, device="cuda")
    tsb.attention_fwd(qkv, out, lse, B, T, NH, hd)
    return qkv, out, dout, lse


@pytest.mark.parametrize("dtype,hd", [(torch.bfloat16, 64), (torch.float32, 32)])
def test_noalloc_matches_allocating_entry_point_twice(dtype, hd):
    # The two entry points run the same deterministic kernels on the same inputs, so
    # the gradients must be bitwise equal; any stale or aliased scratch would show.
    for call, (B, T, NH) in enumerate([(2, 200, 3), (1, 96, 2)]):  # two calls in a row, new shapes
        qkv, out, dout, lse = _inputs(B, T, NH, hd, dtype, seed=10 + call)
        ref = torch.zeros_like(qkv)
        tsb.attention_bwd(qkv, out, dout, lse, ref, B, T, NH, hd)
        got = torch.full_like(qkv, float("nan"))
        tsb.attention_bwd_noalloc(qkv, out, dout, lse, got, B, T, NH, hd)
        torch.cuda.synchronize()
        assert torch.isfinite(got.float()).all()
        assert torch.equal(got, ref)


def test_noalloc_at_the_full_scratch_size():
    # B*NH*T == 2^20 rows: exactly the fixed scratch array.
    B, T, NH, hd = 16, 1024, 64, 64
    assert B * NH * T == 1 << 20
    qkv, out, dout, lse = _inputs(B, T, NH, hd, torch.bfloat16, seed=21)
    ref = torch.zeros_like(qkv)
    tsb.attention_bwd(qkv, out, dout, lse, ref, B, T, NH, hd)
    got = torch.full_like(qkv, float("nan"))
    tsb.attention_bwd_noalloc(qkv, out, dout, lse, got, B, T, NH, hd)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    B, T, NH, hd = 1, 1, 1, 64
    qkv, out, dout, lse = _inputs(B, T, NH, hd, torch.bfloat16, seed=3)
    dq = torch.zeros_like(qkv)
    with pytest.raises(tsb.Gpt2Error) as e:
        # B*NH*T = 2^20 + 1 rows: rejected before any kernel is launched
        tsb.lib()  # loaded
        code = tsb.lib().gpt2_op_attention_bwd_noalloc(tsb.BF16, qkv.data_ptr(), out.data_ptr(), dout.data_ptr(),
                                                       lse.data_ptr(), 1, (1 << 20) + 1, 1, 64, dq.data_ptr(),
                                                       torch.cuda.current_stream().cuda_stream)
        tsb._op(code)
    assert e.value.code == -1
    assert "exceeds the fixed scratch" in str(e.value)
