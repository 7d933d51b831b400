"""Host-side argument checks of the Python binding: the C ABI receives
pointers only, so shapes and extents are checked before any launch."""
import pytest
import torch

from matrix_aware_optimizers_muon_b200 import _check_extent, _check_state_shapes


class _Dev:
    """Stands in for a contiguous CUDA tensor (no GPU here)."""

    def __init__(self, numel, dtype=torch.bfloat16):
        self.is_cuda = True
        self.dtype = dtype
        self._n = numel

    def is_contiguous(self):
        return True

    def numel(self):
        return self._n


def test_extent_accepts_exact_fit_and_padding():
    # 3 matrices of 5 x 7 with row stride 8 and matrix stride 40
    _check_extent(_Dev(2 * 40 + 4 * 8 + 7), "A", 5, 7, 8, 40, 3, (torch.bfloat16,))
    _check_extent(_Dev(5 * 7), "A", 5, 7, 7, 0, 1, (torch.bfloat16,))


def test_extent_rejects_short_tensor_and_bad_ld_and_dtype():
    with pytest.raises(ValueError, match="needs"):
        _check_extent(_Dev(2 * 40 + 4 * 8 + 6), "A", 5, 7, 8, 40, 3, (torch.bfloat16,))
    with pytest.raises(ValueError, match="leading dimension"):
        _check_extent(_Dev(10 ** 6), "B", 5, 7, 6, 40, 1, (torch.bfloat16,))
    with pytest.raises(ValueError, match="dtype"):
        _check_extent(_Dev(10 ** 6, torch.float16), "D", 5, 7, 8, 40, 1, (torch.bfloat16, torch.float32))
    with pytest.raises(ValueError, match="dtype"):
        _check_extent(torch.zeros(100, dtype=torch.bfloat16), "A", 2, 2, 2, 0, 1, (torch.bfloat16,))


def test_soap_state_shapes():
    m, n = 6, 10
    ok = dict(W=torch.zeros(m, n), G=torch.zeros(m, n), M=torch.zeros(m, n), V=torch.zeros(m, n),
              L=torch.zeros(m, m), QL=torch.zeros(m, m), R=None, QR=None)
    _check_state_shapes(0, ok, ("G", "M", "V"))
    for k, bad in (("V", torch.zeros(n, m)), ("G", torch.zeros(m, n + 1)), ("QL", torch.zeros(n, n)),
                   ("R", torch.zeros(m, m)), ("QR", torch.zeros(n, m))):
        d = dict(ok, **{k: bad})
        with pytest.raises(ValueError, match=k):
            _check_state_shapes(3, d, ("G", "M", "V"))
    with pytest.raises(ValueError, match="2-D"):
        _check_state_shapes(0, dict(ok, W=torch.zeros(m * n)), ("G", "M", "V"))


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """No CPU fallback: without libmo.so the binding refuses to load."""
    from matrix_aware_optimizers_muon_b200 import _lib
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "libmo.so"))
    with pytest.raises(ImportError, match="no CPU fallback"):
        _lib.load()
