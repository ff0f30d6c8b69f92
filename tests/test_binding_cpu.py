"""The tensor-level Python entries refuse what the library cannot take, on a
machine without a GPU: CPU tensors, wrong shapes, mixed dtypes,
non-contiguous views and wrong table or weight shapes raise before any CUDA
call.  Nothing is ever computed on the CPU instead: there is no fallback."""
import pytest
import torch

from vit_bidirectional_attention_b200 import vitattn


def bf16(*shape):
    return torch.zeros(*shape, dtype=torch.bfloat16)


def test_forward_rejects_cpu_tensors_instead_of_computing():
    q = bf16(1, 64, 2, 64)
    with pytest.raises(ValueError, match="CUDA"):
        vitattn.forward(q, q.clone(), q.clone())


@pytest.mark.parametrize("k_shape,v_shape", [((1, 64, 2, 32), (1, 64, 2, 64)), ((1, 64, 2, 64), (1, 32, 2, 64))])
def test_forward_rejects_mismatched_shapes(k_shape, v_shape):
    with pytest.raises(ValueError, match="shape"):
        vitattn.forward(bf16(1, 64, 2, 64), bf16(*k_shape), bf16(*v_shape))


def test_forward_rejects_a_three_dimensional_query():
    q = bf16(64, 2, 64)
    with pytest.raises(ValueError):
        vitattn.forward(q, q, q)


def test_varlen_rejects_cpu_tensors_and_bad_shapes():
    q = bf16(96, 2, 64)
    with pytest.raises(ValueError, match="CUDA"):
        vitattn.forward_varlen(q, q.clone(), q.clone(), [0, 40, 96])
    with pytest.raises(ValueError, match="shape"):
        vitattn.forward_varlen(q, bf16(96, 2, 32), q.clone(), [0, 96])


def test_gqa_rejects_cpu_tensors_and_bad_kv_shapes():
    q = bf16(1, 64, 8, 64)
    kv = bf16(1, 64, 2, 64)
    with pytest.raises(ValueError, match="CUDA"):
        vitattn.forward_gqa(q, kv, kv.clone())
    with pytest.raises(ValueError):
        vitattn.forward_gqa(q, kv, bf16(1, 64, 4, 64))      # k and v differ
    with pytest.raises(ValueError):
        vitattn.forward_gqa(q, bf16(1, 32, 2, 64), bf16(1, 32, 2, 64))   # token counts differ


def test_ext_rejects_cpu_tensors_and_bad_shapes():
    q = bf16(1, 64, 2, 64)
    kv = bf16(1, 96, 2, 64)
    with pytest.raises(ValueError, match="CUDA"):
        vitattn.forward_ext(q, kv, kv.clone(), causal=True, with_lse=True)
    with pytest.raises(ValueError):
        vitattn.forward_ext(q, bf16(1, 96, 3, 64), bf16(1, 96, 3, 64))   # head counts differ


def test_prologues_reject_cpu_tensors_and_bad_shapes():
    qkv = bf16(16, 3, 2, 64)
    cs = torch.zeros(16, 64)
    w = torch.ones(64)
    with pytest.raises(ValueError, match="CUDA"):
        vitattn.qkv_rope(qkv, cs, cs.clone())
    with pytest.raises(ValueError, match="CUDA"):
        vitattn.qkv_norm_rope(qkv, cs, cs.clone(), w, w.clone(), 1e-6)
    with pytest.raises(ValueError):
        vitattn.qkv_rope(bf16(16, 2, 2, 64), cs, cs.clone())         # not q | k | v
    with pytest.raises(ValueError):
        vitattn.qkv_norm_rope(bf16(16, 4, 2, 64), cs, cs.clone(), w, w.clone(), 1e-6)


def test_non_contiguous_views_are_refused_not_copied():
    q = bf16(1, 64, 2, 128)[..., ::2]
    assert not q.is_contiguous()
    with pytest.raises(ValueError):
        vitattn.forward(q, q, q)


def test_unsupported_dtype_is_a_type_error():
    with pytest.raises(TypeError):
        vitattn._dtype_code(torch.zeros(4, dtype=torch.float32))
    assert vitattn._dtype_code(torch.zeros(4, dtype=torch.bfloat16)) == vitattn.BF16
    assert vitattn._dtype_code(torch.zeros(4, dtype=torch.float16)) == vitattn.F16


def test_status_errors_carry_their_code_and_text():
    e = vitattn.VitAttnError(-9, "vitattn_qkv_norm_rope")
    assert e.status == -9 and "vitattn_qkv_norm_rope" in str(e) and "finite" in str(e)


def test_tensors_on_different_devices_are_refused():
    # every wrapper calls this check after its shape checks and before the
    # library; a tensor on another device than the first one raises
    a = torch.zeros(4)
    b = torch.zeros(4, device="meta")
    vitattn._same_device("t", a, a.clone(), a.clone())
    with pytest.raises(ValueError, match="device"):
        vitattn._same_device("t", a, a.clone(), b)


def test_a_stream_of_another_device_is_refused():
    class FakeStream:
        device = torch.device("cuda", 1)
        cuda_stream = 1234

    assert vitattn._stream_handle(77, torch.device("cuda", 0)) == 77
    assert vitattn._stream_handle(FakeStream(), torch.device("cuda", 1)) == 1234
    with pytest.raises(ValueError, match="stream"):
        vitattn._stream_handle(FakeStream(), torch.device("cuda", 0))
