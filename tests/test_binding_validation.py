"""The Python binding's own argument checks, on the CPU: each raises ValueError
before anything reaches the library or the GPU (CPU tensors and host arrays
are rejected where device memory is required)."""
import numpy as np
import pytest
import torch


@pytest.fixture(scope="module")
def cq():
    from minimax_scale_search_b200 import build
    build.build()
    from minimax_scale_search_b200 import cq as binding
    return binding


def test_selection_rejects_bad_arguments(cq):
    W = torch.zeros((4, 128), dtype=torch.int16)
    D = torch.ones((2, 128), dtype=torch.float32)
    with pytest.raises(ValueError, match="CUDA"):
        cq.select_scales(W, D)
    with pytest.raises(ValueError, match="2-D"):
        cq._shapes(torch.zeros((4, 100), dtype=torch.int16), D, None)
    with pytest.raises(ValueError, match="K does not match"):
        cq._shapes(W, D, 256)
    with pytest.raises(ValueError, match=r"\[E, G, 128\]"):
        cq._shapes(W, torch.ones((2, 3, 128)), None)
    with pytest.raises(ValueError, match=r"\[E, K\]"):
        cq._shapes(W, torch.ones(128), None)
    assert cq._shapes(W, D, None) == (4, 2, 128)
    assert cq._shapes(W, torch.ones((3, 4, 128)), None) == (4, 3, 0)


def test_host_entry_point_rejects_bad_arrays(cq):
    D = np.ones((2, 128), dtype=np.float32)
    with pytest.raises(ValueError, match="16-bit"):
        cq.select_scales_host(np.zeros((4, 128), dtype=np.float32), D)
    with pytest.raises(ValueError, match="16-bit"):
        cq.select_scales_host(np.zeros((4, 100), dtype=np.uint16), D)
    with pytest.raises(ValueError, match="float32"):
        cq.select_scales_host(np.zeros((4, 128), dtype=np.uint16), D.astype(np.float64))
    with pytest.raises(ValueError, match="16-bit"):
        cq.select_scales_host(np.zeros((128, 8), dtype=np.uint16).T, D)  # not contiguous


def test_policy_and_format_entry_points_reject_bad_arguments(cq):
    W = torch.zeros((4, 128), dtype=torch.int16)
    with pytest.raises(ValueError, match="CUDA"):
        cq.absmax_scales(W)
    with pytest.raises(ValueError, match="CUDA"):
        cq.pool_diagonals(torch.ones((2, 128)))
    with pytest.raises(ValueError, match="unknown policy"):
        cq.policy_scales("minmax", W, torch.ones((2, 128)))
    with pytest.raises(ValueError, match="R\\*K/128"):
        cq.gptq_export(torch.zeros(3, dtype=torch.int16), torch.zeros((4, 16), dtype=torch.int32), 8, 128)
    with pytest.raises(ValueError, match="CUDA"):
        cq.select_scales_spec(W, torch.ones((2, 128)), qmin=-4, qmax=3)
    with pytest.raises(ValueError, match="CUDA"):
        cq.estimate_diagonals(torch.zeros((8, 128), dtype=torch.bfloat16), np.array([0, 4, 8]))


def test_proxy_rejects_offsets_outside_the_groups(cq):
    if not torch.cuda.is_available():
        # the offsets are checked on the host before any device work; with no
        # GPU the per_env tensor itself is refused first
        with pytest.raises(ValueError):
            cq.reconstruction_proxy(torch.zeros((4, 2), dtype=torch.float64), np.array([0, 2, 5]))
        return
    pe = torch.zeros((4, 2), dtype=torch.float64, device="cuda")
    with pytest.raises(ValueError, match="offsets"):
        cq.reconstruction_proxy(pe, np.array([0, 2, 5]))
    with pytest.raises(ValueError, match="offsets"):
        cq.reconstruction_proxy(pe, np.array([0, 3, 2, 4]))
