"""CPU checks of the torch helpers' argument validation.

attention_forward / attention_backward hand raw pointers to the C ABI, which
cannot see dtypes, strides or devices.  So the helpers check every tensor
(shape, then dtype, then contiguity, then one CUDA device) and raise
AxisAttnError before any library call; on this CPU-only machine a correct call
therefore stops at the device check, and each wrong one must stop earlier with
its own message.
"""
import pytest
import torch

import causal_attention_fwd_b200 as aa

B, S, Hq, Hkv, D = 1, 8, 4, 2, 64


def bf(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def qkv():
    return bf(B, S, Hq, D), bf(B, S, Hkv, D), bf(B, S, Hkv, D)


def fwd_error(*args, **kw):
    with pytest.raises(aa.AxisAttnError) as e:
        aa.attention_forward(*args, **kw)
    return e.value


def bwd_error(**over):
    q, k, v = qkv()
    a = dict(q=q, k=k, v=v, o=bf(B, S, Hq, D), lse=torch.zeros(B, Hq, S), dout=bf(B, S, Hq, D))
    a.update(over)
    with pytest.raises(aa.AxisAttnError) as e:
        aa.attention_backward(a["q"], a["k"], a["v"], a["o"], a["lse"], a["dout"],
                              grads=over.get("grads"), workspace=over.get("workspace"))
    return e.value


def test_correct_cpu_call_stops_at_the_device_check():
    e = fwd_error(*qkv())
    assert e.code == 4 and "CUDA device" in str(e)
    e = bwd_error()
    assert e.code == 4 and "CUDA device" in str(e)


def test_forward_rejects_wrong_dtype():
    q, k, v = qkv()
    e = fwd_error(q.float(), k, v)
    assert e.code == 4 and "q is torch.float32" in str(e)
    e = fwd_error(q, k.half(), v)
    assert "k is torch.float16" in str(e)


def test_forward_rejects_non_contiguous():
    q, k, v = qkv()
    qt = bf(B, Hq, S, D).transpose(1, 2)  # right shape, wrong strides
    e = fwd_error(qt, k, v)
    assert e.code == 3 and "contiguous" in str(e)


def test_forward_rejects_shape_mismatches():
    q, k, v = qkv()
    assert "Hq = 4 is not a multiple of Hkv = 3" in str(fwd_error(q, bf(B, S, 3, D), bf(B, S, 3, D)))
    assert "v has shape" in str(fwd_error(q, k, bf(B, S + 1, Hkv, D)))
    assert "k has shape" in str(fwd_error(q, bf(B, S, Hkv, D // 2), v))
    assert "4-D" in str(fwd_error(q[0], k, v))
    e = fwd_error(q, k, v, lse=torch.zeros(B, Hq, S + 1))
    assert "lse has shape" in str(e)
    e = fwd_error(q, k, v, out=bf(B, S, Hq, D).float())
    assert "out is torch.float32" in str(e)


def test_backward_rejects_each_bad_tensor():
    assert "o has shape" in str(bwd_error(o=bf(B, S, Hkv, D)))
    assert "dout is torch.float32" in str(bwd_error(dout=torch.zeros(B, S, Hq, D)))
    assert "lse is torch.bfloat16" in str(bwd_error(lse=bf(B, Hq, S)))
    grads = (bf(B, S, Hq, D), bf(B, S, Hq, D), bf(B, S, Hkv, D))
    assert "dk has shape" in str(bwd_error(grads=grads))
    assert "grads must be" in str(bwd_error(grads=grads[:2]))
    ws = torch.zeros(64, dtype=torch.uint8)[::2]
    assert "workspace must be a contiguous" in str(bwd_error(workspace=ws))


def test_mixed_devices_are_rejected_before_any_call():
    # a 'meta' tensor stands in for a second device: the check compares devices
    q, k, v = qkv()
    e = fwd_error(q, k, torch.empty((B, S, Hkv, D), dtype=torch.bfloat16, device="meta"))
    assert e.code == 4  # the first tensor is not on CUDA


def dec_error(layout="NHD", **over):
    a = dict(q=bf(2, 8, D), k_cache=bf(5, 16, 4, D), v_cache=bf(5, 16, 4, D),
             block_table=torch.zeros(2, 3, dtype=torch.int32), seq_lens=torch.ones(2, dtype=torch.int32))
    a.update(over)
    with pytest.raises(aa.AxisAttnError) as e:
        aa.attention_decode(a["q"], a["k_cache"], a["v_cache"], a["block_table"], a["seq_lens"], layout=layout)
    return e.value


def test_decode_layouts_read_the_cache_shape_their_own_way():
    # [num_pages, page_size, Hkv, D] and [num_pages, Hkv, page_size, D] of the same pool
    e = dec_error("NHD")
    assert e.code == 4 and "CUDA device" in str(e)
    e = dec_error("HND", k_cache=bf(5, 4, 16, D), v_cache=bf(5, 4, 16, D))
    assert e.code == 4 and "CUDA device" in str(e)
    # v_cache in the other layout than k_cache
    e = dec_error("HND", k_cache=bf(5, 4, 16, D))
    assert "v_cache" in str(e)
    e = dec_error("BHSD")
    assert "layout" in str(e)


def test_decode_several_tokens_checks_shapes():
    # q [B, q_len, Hq, D]: correct shapes stop at the device check, a wrong lse shape earlier
    base = dict(q=bf(2, 3, 8, D), k_cache=bf(5, 16, 4, D), v_cache=bf(5, 16, 4, D),
                block_table=torch.zeros(2, 3, dtype=torch.int32), seq_lens=torch.full((2,), 3, dtype=torch.int32))
    with pytest.raises(aa.AxisAttnError) as e:
        aa.attention_decode(*base.values())
    assert e.value.code == 4 and "CUDA device" in str(e.value)
    with pytest.raises(aa.AxisAttnError) as e:  # lse of a 4-D q is [B, Hq, q_len]
        aa.attention_decode(*base.values(), lse=torch.zeros(2, 8))
    assert "lse" in str(e.value)
    with pytest.raises(aa.AxisAttnError) as e:  # out must be shaped like q
        aa.attention_decode(*base.values(), out=bf(2, 8, D))
    assert "out" in str(e.value)
    with pytest.raises(aa.AxisAttnError) as e:  # a 5-D q is neither form
        aa.attention_decode(bf(2, 3, 1, 8, D), *list(base.values())[1:])
    assert "q must be" in str(e.value)
