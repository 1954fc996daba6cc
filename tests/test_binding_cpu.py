"""Host logic of the Python binding that needs no GPU: which tensor views can be
passed to the strided entry points as they are (dense rows, evenly spaced), and
their row pitch."""
import pytest
import torch

from elementwise_reduction_b200 import row_pitch


def test_row_pitch_of_dense_and_strided_views():
    a = torch.empty(10, 64)
    assert row_pitch(a) == 64                                   # contiguous
    assert row_pitch(a[:, :32]) == 64                           # column slice: pitch of the parent
    assert row_pitch(a[::2]) == 128                             # every other row
    assert row_pitch(a[3:7, 5:9]) == 64                         # a window
    assert row_pitch(torch.empty(4, 5, 64)[:, :, :10]) == 64    # leading dims collapse evenly
    assert row_pitch(torch.empty(3)) == 3                       # one row
    assert row_pitch(torch.empty(1, 5)) == 5
    assert row_pitch(torch.empty(0, 5)) == 5                    # no rows


@pytest.mark.parametrize("view", [
    lambda: torch.empty(32, 8).t(),                  # columns are not dense
    lambda: torch.empty(4, 6, 32)[:, 1:3],           # leading dimensions do not collapse
    lambda: torch.empty(8, 16)[:, ::2],              # strided last dimension
    lambda: torch.empty(16).expand(4, 16),           # rows overlap (pitch 0)
    lambda: torch.empty(()),                         # a scalar has no rows
])
def test_row_pitch_rejects_views_the_kernels_cannot_address(view):
    assert row_pitch(view()) is None
