"""There is one implementation of the path: the native library on a CUDA
device.  Without libwfattn.so the loader fails loudly (ImportError naming the
build command), and host tensors are rejected with an error instead of being
computed some other way."""
import pytest
import torch

from attention_forward_tmem_b200 import _lib, api


@pytest.fixture
def no_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "libwfattn.so"))
    monkeypatch.setattr(_lib, "_lib", None)


def test_loader_raises_without_the_library(no_library):
    with pytest.raises(ImportError, match="attention_forward_tmem_b200.build"):
        _lib.load()


@pytest.mark.parametrize("with_library", [True, False])
def test_host_tensors_are_rejected(with_library, monkeypatch, tmp_path):
    if not with_library:
        monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "libwfattn.so"))
        monkeypatch.setattr(_lib, "_lib", None)
    q = torch.zeros(1, 2, 8, 64, dtype=torch.bfloat16)
    calls = [
        lambda: api.attn_fwd(q, q, q),
        lambda: api.attn_fwd(q, q, q, return_lse=True),
        lambda: api.merge(torch.zeros(2, 1, 2, 8, 64), torch.zeros(2, 1, 2, 8)),
        lambda: api.BlockKVCache.allocate((1, 2, 512, 64), (1, 2, 512, 64), chunk_size=128,
                                          window_size=384, sink_size=128, device="cpu",
                                          dtype=torch.bfloat16),
    ]
    for call in calls:
        with pytest.raises((api.WfError, ImportError)) as e:
            call()
        if isinstance(e.value, api.WfError):
            assert "no CPU path" in str(e.value)
