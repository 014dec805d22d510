"""The torch binding on CPU (no GPU): it marshals arguments and nothing else.

Every compute entry point refuses CPU tensors, wrong dtypes and wrong ranks
before the library is called, so no call can quietly run anywhere but the
CUDA kernels; a missing library that cannot be built raises instead of
falling back; a non-OK status from the library becomes a GDNError that names
it.
"""
import pytest
import torch

import gated_deltanet_linear_chunked_b200 as gdn
from gated_deltanet_linear_chunked_b200 import _lib
from gated_deltanet_linear_chunked_b200 import build as _build

B, T, H, D = 1, 8, 2, 16


def scan_args(dtype=torch.bfloat16, device="cpu"):
    q = torch.zeros(B, T, H, D, dtype=dtype, device=device)
    g = torch.zeros(B, T, H, dtype=torch.float32, device=device)
    return q, q.clone(), q.clone(), g, g.clone()


SCANS = ["chunk_fwd", "chunk_bidir", "chunk_fwd_logits", "chunk_bidir_logits"]
BACKWARDS = ["chunk_fwd_backward", "chunk_bidir_backward"]


@pytest.mark.parametrize("name", SCANS)
def test_scans_refuse_cpu_tensors(name):
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        getattr(gdn, name)(*scan_args())


@pytest.mark.parametrize("name", BACKWARDS)
def test_backwards_refuse_cpu_tensors(name):
    q, k, v, g, beta = scan_args(torch.float32)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        getattr(gdn, name)(q, k, v, g, beta, None, v.clone())


def test_attention_and_reset_refuse_cpu_tensors():
    q = torch.zeros(B, T, H, D, dtype=torch.bfloat16)
    kc = torch.zeros(B, 3, T, H, D, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        gdn.sink_window_attention(q, q, q, kc, kc.clone(), 0, 1, 2)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        gdn.state_reset(torch.zeros(B, H, D, D))


@pytest.mark.parametrize("name", SCANS + BACKWARDS)
def test_unsupported_dtype_and_rank(name):
    fn = getattr(gdn, name)
    extra = (None, torch.zeros(B, T, H, D, dtype=torch.float16)) if name in BACKWARDS else ()
    with pytest.raises(TypeError, match="bfloat16 or float32"):
        fn(*scan_args(torch.float16), *extra)
    q, k, v, g, beta = scan_args()
    with pytest.raises(ValueError, match=r"\[B,T,H,Dk\]"):
        fn(q[0], k, v, g, beta, *extra)


def test_status_becomes_a_named_error():
    _lib.check(_lib.GDN_OK, "x")          # OK is silent
    names = ["GDN_ERR_INVALID_ARG", "GDN_ERR_UNSUPPORTED", "GDN_ERR_ALIAS", "GDN_ERR_CUDA",
             "GDN_ERR_TIMEOUT"]
    for status, name in enumerate(names, start=1):
        with pytest.raises(gdn.GDNError, match=name) as e:
            _lib.check(status, "gdn_chunk_fwd")
        assert e.value.status == status and "gdn_chunk_fwd" in str(e.value)


def test_missing_library_raises_instead_of_falling_back(monkeypatch, tmp_path):
    """With the library absent and nvcc failing, the first call raises; no
    other implementation is tried."""
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_build, "LIB_PATH", str(tmp_path / "libgdn.so"))
    monkeypatch.setattr(_build, "is_stale", lambda: True)

    def no_nvcc():
        raise OSError("nvcc not found")
    monkeypatch.setattr(_build, "build", no_nvcc)
    with pytest.raises(RuntimeError, match="libgdn.so is missing"):
        _lib.load()
