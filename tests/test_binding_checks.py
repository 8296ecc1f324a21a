"""The Python binding's checks on caller-supplied buffers, on CPU.  The
kernels read and write through raw pointers, so every buffer must have
exactly the size the call implies; the binding refuses anything else before
a launch.  The checks do not depend on the device type, so CPU tensors
exercise them here."""
import pytest
import torch

import exact_io_aware_65_b200 as fa

CPU = torch.device("cpu")


def test_buffer_of_the_right_size_passes():
    t = torch.empty((2, 3, 300, 64), dtype=torch.bfloat16)
    assert fa._check_buf(t, "O", (2, 3, 300, 64), torch.bfloat16, CPU) is t


@pytest.mark.parametrize("bad", [
    torch.empty((2, 3, 299, 64), dtype=torch.bfloat16),          # one row short
    torch.empty((2, 3, 300, 64), dtype=torch.float32),           # wrong type
    torch.empty((2, 3, 64, 300), dtype=torch.bfloat16).transpose(2, 3),   # right shape, not contiguous
    torch.empty((2 * 3 * 300 * 64,), dtype=torch.bfloat16),      # right size, wrong shape
])
def test_buffer_of_another_size_type_or_layout_is_refused(bad):
    with pytest.raises(fa.FAError) as e:
        fa._check_buf(bad, "O", (2, 3, 300, 64), torch.bfloat16, CPU)
    assert e.value.code == 1


def test_buffer_on_another_device_is_refused():
    t = torch.empty((4,), dtype=torch.float32, device="meta")
    with pytest.raises(fa.FAError):
        fa._check_buf(t, "LSE", (4,), torch.float32, CPU)


def test_workspace_counts_bytes_not_elements():
    need = 1000
    ptr, nbytes = fa._workspace(torch.empty(250, dtype=torch.float32), need, CPU)
    assert nbytes == 1000 and ptr != 0
    with pytest.raises(fa.FAError) as e:
        fa._workspace(torch.empty(999, dtype=torch.uint8), need, CPU)
    assert e.value.code == 4
    with pytest.raises(fa.FAError):
        fa._workspace(torch.empty(4000, dtype=torch.uint8)[::2], need, CPU)   # strided


def test_block_mask_must_cover_the_tile_grid():
    # the kernels read a row-major [nbq, nbk] grid; the binding only sees
    # that on CUDA tensors, so a CPU mask is refused first
    with pytest.raises(fa.FAError):
        fa._mask("block", torch.ones((3, 3), dtype=torch.uint8), 3, 3, CPU)
    with pytest.raises(fa.FAError):
        fa._mask("block", None, 3, 3, CPU)
    assert fa._mask("causal", None, 3, 3, CPU) == (1, None)
    assert fa._mask("none", torch.ones(1), 3, 3, CPU) == (0, None)     # ignored for other kinds


def test_entry_points_refuse_host_tensors_before_any_launch():
    q = torch.zeros((1, 1, 128, 64), dtype=torch.bfloat16)
    with pytest.raises(fa.FAError):
        fa.fwd(q, q, q)
    with pytest.raises(fa.FAError):
        fa.bwd(q, q, q, q, q, torch.zeros((1, 1, 128)))
    with pytest.raises(fa.FAError):
        fa.decode(q[:, :, :1], q, q)
    with pytest.raises(fa.FAError):
        fa.standard_fwd(q, q, q)


def test_tile_counts():
    assert [fa._tiles(n) for n in (1, 127, 128, 129, 8192)] == [1, 1, 1, 2, 64]
