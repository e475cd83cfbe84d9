"""Helpers shared by the GPU tests (no layer arithmetic here)."""
import numpy as np
import pytest
import torch

from transformer_layer_step_b200 import gptlayer as G
from transformer_layer_step_b200 import synth
from transformer_layer_step_b200.harness import TORCH_DT, bits_to_tensor, tensor_to_bits


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def dev_tensor(values: np.ndarray, dtype: str) -> torch.Tensor:
    """float64 values -> device tensor of the 16-bit type (RNE)."""
    return bits_to_tensor(synth.to_bits(values, dtype), dtype, "cuda")


def host_values(t: torch.Tensor, dtype: str) -> np.ndarray:
    return synth.from_bits(tensor_to_bits(t), dtype).reshape(t.shape)


def rounded(values: np.ndarray, dtype: str) -> np.ndarray:
    return synth.from_bits(synth.to_bits(values, dtype), dtype).reshape(values.shape)


def stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def check_device_error():
    torch.cuda.synchronize()
    word = G.read_device_error(clear=True)
    assert word == 0, f"device error word {word:#x}"


def rel_max_err(got: np.ndarray, ref: np.ndarray) -> float:
    rms = float(np.sqrt(np.mean(ref.astype(np.float64) ** 2)))
    return float(np.abs(got.astype(np.float64) - ref).max()) / max(rms, 1e-30)
