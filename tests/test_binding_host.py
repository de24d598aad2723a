"""The Python binding without a GPU: it has no fallback.  A missing library
is an ImportError at first use, every C-ABI signature it declares is
exported by the built library, and calls are refused (not emulated) on a
machine without a usable sm_100 device."""
import os

import pytest
import torch

import long_context_bidirectional_b200 as b2a


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(b2a, "_LIB_PATH", str(tmp_path / "nowhere" / "libb200attn.so"))
    monkeypatch.setattr(b2a, "_lib", None)
    with pytest.raises(ImportError, match="not found"):
        b2a._get_lib()


def test_every_binding_signature_is_exported():
    if not os.path.exists(b2a.library_path()):
        pytest.skip("library not built")
    lib = b2a._get_lib()
    for name in b2a._SIGS:
        assert hasattr(lib, name), name


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU refusal")
def test_calls_are_refused_without_a_device():
    if not os.path.exists(b2a.library_path()):
        pytest.skip("library not built")
    # a valid-looking call reaches the device check and fails with a status,
    # instead of running anything on the CPU
    lib = b2a._get_lib()
    fake = 0x10000
    st = lib.attn_fwd(fake, fake, fake, fake, None, 256, 2, 64, 0.125, 128, 128, 128, 128, None)
    assert st in (2, 3)   # unsupported device / CUDA error
    st = lib.qkv_proj(fake, fake, fake, 128, 256, 64, None)
    assert st in (2, 3)
