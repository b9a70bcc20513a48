"""The torch wrappers refuse mismatched tensors before calling the library
(no GPU needed: every case fails on the host)."""
import pytest
import torch

from gated_delta_rule_147_b200 import TIED, chunk_bwd, chunk_fwd, decode_step


def t(*shape, dtype=torch.bfloat16):
    return torch.zeros(shape, dtype=dtype)


def test_chunk_fwd_dtype_mismatch():
    with pytest.raises(TypeError, match="v has dtype"):
        chunk_fwd(t(1, 8, 2, 16), t(1, 8, 2, 16), t(1, 8, 2, 16, dtype=torch.float32))
    with pytest.raises(TypeError, match="alpha has dtype"):
        chunk_fwd(t(1, 8, 2, 16), t(1, 8, 2, 16), t(1, 8, 2, 16), t(1, 8, 2, dtype=torch.float32))
    with pytest.raises(TypeError, match="S0 has dtype"):
        chunk_fwd(t(1, 8, 2, 16), t(1, 8, 2, 16), t(1, 8, 2, 16), None, None, None,
                  t(1, 2, 16, 16))
    with pytest.raises(TypeError, match="unsupported dtype"):
        chunk_fwd(t(1, 8, 2, 16, dtype=torch.float16), t(1, 8, 2, 16), t(1, 8, 2, 16))


def test_host_tensors_are_refused():
    with pytest.raises(ValueError, match="CUDA tensors"):
        chunk_fwd(t(1, 8, 2, 16), t(1, 8, 2, 16), t(1, 8, 2, 16), t(1, 8, 2), t(1, 8, 2), TIED)
    with pytest.raises(ValueError, match="CUDA tensors"):
        decode_step(t(2, 2, 16), t(2, 2, 16), t(2, 2, 16), None, None, None,
                    t(2, 2, 16, 16, dtype=torch.float32))
    with pytest.raises(ValueError, match="CUDA tensors"):
        chunk_bwd(t(1, 8, 2, 16), t(1, 8, 2, 16), t(1, 8, 2, 16), dO=t(1, 8, 2, 16))


def test_chunk_bwd_dtype_mismatch():
    with pytest.raises(TypeError, match="dO has dtype"):
        chunk_bwd(t(1, 8, 2, 16), t(1, 8, 2, 16), t(1, 8, 2, 16), dO=t(1, 8, 2, 16, dtype=torch.float32))
    with pytest.raises(TypeError, match="dS_T has dtype"):
        chunk_bwd(t(1, 8, 2, 16), t(1, 8, 2, 16), t(1, 8, 2, 16), dO=t(1, 8, 2, 16),
                  dS_T=t(1, 2, 16, 16))


def test_decode_state_must_be_fp32():
    with pytest.raises(TypeError, match="S has dtype"):
        decode_step(t(2, 2, 16), t(2, 2, 16), t(2, 2, 16), None, None, None, t(2, 2, 16, 16))
